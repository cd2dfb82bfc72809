// Persistent split-K tcgen05 GEMM with fused epilogues (see gemm.cuh).
//
// CTA = 8 warps:  warp 0 lane 0 issues TMA loads of (weight tile, token tile)
// pairs into an S-stage shared-memory ring; warp 1 lane 0 issues tcgen05.mma
// (M=128, N=NT, K=16, bf16 in, fp32 accumulate) into one of two TMEM
// accumulator buffers; warps 2..5 (128 threads, one TMEM lane each) drain a
// finished accumulator with tcgen05.ld, resolve split tiles, and run the
// epilogue while the next tile accumulates in the other buffer; warps 6 and 7,
// when the GEMM consumes RMS-normalised rows, rewrite each token tile in shared
// memory as R(x * inv_rms * gain) between its arrival and the MMA.
#include <algorithm>

#include "gemm.cuh"

namespace df {

// Largest grid the launcher is given (the C ABI caps it at 160 CTAs).
constexpr long long kGemmMaxGrid = 160;

// Tile configuration per token width NT: one CTA per SM with the deepest ring
// that fits (two CTAs per SM with half the ring measured slower at batch 1).
template <int NT, bool CLU = false>
struct GemmCfg {
    static constexpr int THREADS = 256;
    static constexpr bool TWO_PER_SM = false;
    static constexpr int A_BYTES = 128 * 128;            // 128 rows x 64 bf16
    static constexpr int B_BYTES = NT * 128;             // NT rows x 64 bf16
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int CH = NT < 32 ? NT : 32;         // epilogue column chunk
    static constexpr int XCH_FLOATS = 128 * (CH + 1);
    static constexpr int GAIN_MAX = 4096;                // RMSNorm gain elements staged in shared memory
    static constexpr int MISC_BYTES = 6144 + GAIN_MAX * 2;
    // Cluster mode (its own instance, so the whole-grid kernel keeps the deeper ring):
    // the partials of up to 3 peers of the cluster land here, rows padded to NT + 4
    // floats so 16-byte reads of a row are conflict-free.
    static constexpr int LAND_SLOTS = CLU ? 3 : 0;
    static constexpr int LAND_LD = NT + 4;
    static constexpr int LAND_BYTES = LAND_SLOTS * 128 * LAND_LD * 4;
    static constexpr int SMEM_CAP = TWO_PER_SM ? (233472 / 2 - 2048) : 232448;
    static constexpr int BUDGET = SMEM_CAP - 1024 - XCH_FLOATS * 4 - LAND_BYTES - MISC_BYTES;
    static constexpr int STAGES_RAW = BUDGET / STAGE_BYTES;
    static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
    static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + XCH_FLOATS * 4 + LAND_BYTES + MISC_BYTES;
    static constexpr uint32_t TMEM_COLS = (2 * NT < 32) ? 32 : 2 * NT;
    static constexpr int MIN_BLOCKS = TWO_PER_SM ? 2 : 1;
};

DF_DEV float silu(float g) { return g / (1.0f + expf(-g)); }

// The work partition of gemm.cuh in 32-bit arithmetic, for U * P < 2^32 (the
// launcher checks): the split-tile bookkeeping sits on the critical path of a
// GEMM's last tiles, where 64-bit divisions cost.
DF_DEV uint32_t sk32_begin(uint32_t p, uint32_t U, uint32_t P) { return p * U / P; }
DF_DEV uint32_t sk32_owner(uint32_t u, uint32_t U, uint32_t P) { return ((u + 1) * P - 1) / U; }

// Weighted whole-grid partition: CTAs [L, P) take d units fewer than CTAs [0, L).
// With E = U + (P - L) d, begin(p) = floor((p E - max(0, p - L) d P) / P), so the
// early CTAs own E / P units each and the late ones (U - L d) / P; the launcher
// keeps U - L d >= P and P E < 2^32.  owner(u) is the largest p with begin(p) <= u.
DF_DEV uint32_t skw32_begin(uint32_t p, uint32_t U, uint32_t P, uint32_t L, uint32_t d) {
    const uint32_t E = U + (P - L) * d;
    return (p * E - (p > L ? p - L : 0u) * d * P) / P;
}
DF_DEV uint32_t skw32_owner(uint32_t u, uint32_t U, uint32_t P, uint32_t L, uint32_t d) {
    const uint32_t E = U + (P - L) * d;
    const uint32_t pe = ((u + 1) * P - 1) / E;
    if (pe < L) return pe;
    const uint32_t pl = ((u + 1) * P - L * d * P - 1) / (U - L * d);
    return pl < P - 1 ? pl : P - 1;
}

// Top-2 merge: a <- top2(a ∪ b); ties of the top value go to the lower id.
DF_DEV void top2_merge(float& a1, int& ai, float& a2, float b1, int bi, float b2) {
    if (b1 > a1 || (b1 == a1 && bi < ai)) {
        a2 = fmaxf(a1, b2);
        a1 = b1;
        ai = bi;
    } else {
        a2 = fmaxf(a2, b1);
    }
}

// What the producer warp copies into the idle ring for the finishing epilogue of a
// wide tile (posted by the epilogue once the tile's accumulator and the peers'
// partials are ready; depth 0: nothing).
struct LandPlan {
    int depth;                 // chunk buffers in flight (0: no landing)
    int nchunks;               // CH-token chunks of the tile
    int lbuf;                  // bytes per chunk buffer
    int n_peer;                // peers' partial chunks per buffer (first, 16 KB each)
    int aux;                   // 0 none, 1 residual rows (tensor tile), 2 RoPE rows of the chunk's tokens
    int aux_row;               // aux bytes per token
    int tx_x, tx_y0;           // residual tile coordinates of chunk 0
    const float* psrc[12];     // the peers' partials of this tile
};

template <int NT, bool CLU>
__global__ void __launch_bounds__(GemmCfg<NT, CLU>::THREADS, GemmCfg<NT, CLU>::MIN_BLOCKS)
    k_gemm_tc(const __grid_constant__ GemmParams p) {
    using C = GemmCfg<NT, CLU>;
    constexpr int S = C::STAGES;
    constexpr int CH = C::CH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align_up<uint8_t>(smem_raw, 1024);
    uint8_t* sA = smem;
    uint8_t* sB = smem + S * C::A_BYTES;
    float* xch = (float*)(sB + S * C::B_BYTES);
    __nv_bfloat16* const xout = (__nv_bfloat16*)xch;   // epilogue outputs, token-major [CH][128] bf16
    float* land = xch + C::XCH_FLOATS;                 // [LAND_SLOTS][128][LAND_LD] peers' partials
    uint64_t* full = (uint64_t*)(land + C::LAND_BYTES / 4);
    uint64_t* empty = full + S;
    uint64_t* accf = empty + S;
    uint64_t* acce = accf + 2;
    uint64_t* drain = acce + 2;
    uint64_t* landb = drain + 1;      // cluster mode: the peers' partials have landed
    uint64_t* landc = landb + 1;      // [3] chunked landing: chunk buffer filled (NT >= 64)
    uint64_t* lfree = landc + 3;      // [3] chunked landing: chunk buffer consumed by the epilogue
    uint64_t* land_go = lfree + 3;    // chunked landing: the plan is posted
    uint32_t* tmem_slot = (uint32_t*)(land_go + 1);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
    int* s_flag = (int*)(tmem_slot + 2);
    int* tok_b = s_flag + 1;          // [NT]
    int* tok_pos = tok_b + NT;        // [NT]
    float* inv_s = (float*)(tok_pos + NT);   // [2][NT] inverse RMS of the current m-tile's rows, per normaliser warp
    uint64_t* ready = smem_align_up<uint64_t>(inv_s + 2 * NT, 8);   // [S] normalised B stages
    __nv_bfloat16* sgain = smem_align_up<__nv_bfloat16>(ready + S, 16);   // [GAIN_MAX]
    LandPlan* plan = smem_align_up<LandPlan>(sgain + C::GAIN_MAX, 16);
    static_assert((2 * S + 13) * 8 + 16 + 2 * NT * 4 + 2 * NT * 4 + 8 + S * 8 + 16 + C::GAIN_MAX * 2 + 16 +
                          (int)sizeof(LandPlan) <=
                      C::MISC_BYTES, "misc");

    // shared-window addresses of what the epilogues read back
    const uint32_t xch_a = smem_u32(xch), tok_b_a = smem_u32(tok_b), tok_pos_a = smem_u32(tok_pos);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long* trace = p.trace ? p.trace + (size_t)blockIdx.x * 8 : nullptr;
    const long long clk0 = clock64();
    if (trace && threadIdx.x == 0) trace[0] = (long long)globaltimer_ns();

    // Work partition.  Whole grid: CTA p owns k-block units [pU/P, (p+1)U/P) of all
    // output tiles.  Grouped (several token tiles): CTA p = g * m_tiles + m takes token
    // tile m of group g's share of the (weight tile, k-block) units, so the m_tiles
    // CTAs of a group read each weight tile at about the same time (one HBM read, the
    // others L2 hits) instead of at unrelated offsets.  Cluster mode (CL >= 2):
    // cluster q of Q owns whole tiles [qT/Q, (q+1)T/Q), and its CL CTAs split that
    // cluster's units the same way, so every split tile's contributors are CTAs of
    // one cluster.  rloc is the CTA's index within its partition (group, rank).
    const long long U = p.units;
    const int P = p.ctas, cta = blockIdx.x, KB = p.KB, m_tiles = p.m_tiles;
    const int CL = (CLU && p.cluster >= 2) ? p.cluster : 0;
    // (only the widest token tile ever has several: narrower widths are picked for M <= NT)
    const int GM = (NT == 256 && p.grouped && !CL) ? m_tiles : 1;   // CTAs per group
    const int gm = cta % GM;                                             // the group's token tile
    long long ubase = 0, Uloc = U / GM;
    int Ploc = P / GM, rloc = cta / GM, cbase = 0;
    // global tile of partition unit u, and the CTA of partition index i
    auto tile_of = [&](long long u) -> long long { return GM > 1 ? (u / KB) * m_tiles + gm : u / KB; };
    auto cta_of = [&](int i) -> int { return (cbase + i) * GM + gm; };
    if constexpr (C::LAND_SLOTS > 0) {
        if (CL) {
            const int q = cta / CL, Q = P / CL;
            const long long T = U / KB;
            const long long t0 = T * q / Q, t1 = T * (q + 1) / Q;
            ubase = t0 * KB;
            Uloc = (t1 - t0) * KB;
            Ploc = CL;
            rloc = cta % CL;
            cbase = q * CL;
        }
    }
    // weighted shares (whole grid only)
    const bool WT = p.late_deficit > 0 && GM == 1 && !CL && !p.whole_tiles;
    const uint32_t wL = (uint32_t)p.late_from, wd = (uint32_t)p.late_deficit;
    long long u_begin = ubase + sk_begin(rloc, Uloc, Ploc), u_end = ubase + sk_begin(rloc + 1, Uloc, Ploc);
    if (WT) {
        u_begin = skw32_begin((uint32_t)cta, (uint32_t)U, (uint32_t)P, wL, wd);
        u_end = skw32_begin((uint32_t)cta + 1, (uint32_t)U, (uint32_t)P, wL, wd);
    }
    if (p.whole_tiles && !CL) {   // tile-granular ranges: no tile is split, no partials
        const long long T = Uloc / KB;
        u_begin = (T * rloc / Ploc) * KB;
        u_end = (T * (rloc + 1) / Ploc) * KB;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], 128);
        }
        for (int s2 = 0; s2 < S; ++s2) mbar_init(&ready[s2], 2);   // one arrival per normaliser warp
        mbar_init(drain, 1);
        mbar_init(landb, 1);
        for (int j = 0; j < 3; ++j) {
            mbar_init(&landc[j], 1);
            mbar_init(&lfree[j], 128);
        }
        mbar_init(land_go, 1);
        if (CL) {
            // The CTA's last segment is a split tile it finishes when it starts at the
            // tile's k-block 0 and ends inside it: expect its peers' partials.
            const long long tl = (u_end - 1) / KB;
            if (u_begin <= tl * KB && u_end < (tl + 1) * KB) {
                const int nc = sk_owner((tl + 1) * KB - 1 - ubase, Uloc, Ploc) - sk_owner(tl * KB - ubase, Uloc, Ploc) + 1;
                mbar_arrive_expect_tx(landb, (uint32_t)((nc - 1) * 128 * NT * 4));
            }
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < p.n_amat; ++i) tma_prefetch_desc(&p.ta[i]);
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (CL) {
        // every peer's landing barrier is initialised before any partial is sent
        cluster_arrive();
        cluster_wait();
    }

    griddep_launch();
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // Weights are read once: evict first.  In grouped mode the m_tiles CTAs of a
            // group read each weight tile within a short time of each other, so it stays
            // at normal priority until the last of them has it, and the token tiles, read
            // by every group, are kept ahead of it.
            const uint64_t pol_w = GM > 1 ? make_l2_policy_evict_normal() : make_l2_policy_evict_first();
            const uint64_t pol_b = make_l2_policy_evict_last();
            // Weights never depend on the previous kernel: start streaming the
            // first S weight tiles into the ring, and the next l2_prefetch ones
            // into L2, before waiting for it to finish.
            int pre = 0;
            const int s_pre = (p.pre_stages > 0 && p.pre_stages < S) ? p.pre_stages : S;
            const int n_ahead = s_pre + p.l2_prefetch;
            for (long long u = u_begin, idx = 0; u < u_end && idx < n_ahead;) {
                const long long t = tile_of(u);
                const int kb0 = (int)(u % KB);
                const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
                const int n_tile = (int)(t / m_tiles);
                int mi = 0;
                if (!p.swiglu)
                    while (mi + 1 < p.n_amat && n_tile >= p.amat[mi + 1].tile0) ++mi;
                const int arow = p.swiglu ? n_tile * 64 : (n_tile - p.amat[mi].tile0) * 128;
                for (int kb = kb0; kb < kb1 && idx < n_ahead; ++kb, ++idx) {
                    if (idx < s_pre) {
                        mbar_arrive_expect_tx(&full[pre], C::STAGE_BYTES);
                        uint8_t* a = sA + pre * C::A_BYTES;
                        if (p.swiglu) {
                            tma_load_2d_hint(a, &p.ta[0], &full[pre], kb * 64, arow, pol_w);
                            tma_load_2d_hint(a + 64 * 128, &p.ta[1], &full[pre], kb * 64, arow, pol_w);
                        } else {
                            tma_load_2d_hint(a, &p.ta[mi], &full[pre], kb * 64, arow, pol_w);
                        }
                        ++pre;
                    } else if (p.swiglu) {
                        tma_prefetch_l2_2d(&p.ta[0], kb * 64, arow);
                        tma_prefetch_l2_2d(&p.ta[1], kb * 64, arow);
                    } else {
                        tma_prefetch_l2_2d(&p.ta[mi], kb * 64, arow);
                    }
                }
                u += kb1 - kb0;
            }
            griddep_wait();
            if (trace) trace[1] = (long long)globaltimer_ns();
            int stage = 0;
            uint32_t round = 0;
            long long issued = 0;
            bool ok = true;
            for (long long u = u_begin; u < u_end && ok;) {
                const long long t = tile_of(u);
                const int kb0 = (int)(u % KB);
                const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
                const int n_tile = (int)(t / m_tiles), m_tile = (int)(t % m_tiles);
                int mi = 0;
                if (!p.swiglu)
                    while (mi + 1 < p.n_amat && n_tile >= p.amat[mi + 1].tile0) ++mi;
                const int arow = p.swiglu ? n_tile * 64 : (n_tile - p.amat[mi].tile0) * 128;
                for (int kb = kb0; kb < kb1; ++kb) {
                    uint8_t* a = sA + stage * C::A_BYTES;
                    uint8_t* b = sB + stage * C::B_BYTES;
                    if (issued >= pre) {
                        if (!mbar_wait(&empty[stage], (round & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
                        mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
                        if (p.swiglu) {
                            tma_load_2d_hint(a, &p.ta[0], &full[stage], kb * 64, arow, pol_w);
                            tma_load_2d_hint(a + 64 * 128, &p.ta[1], &full[stage], kb * 64, arow, pol_w);
                        } else {
                            tma_load_2d_hint(a, &p.ta[mi], &full[stage], kb * 64, arow, pol_w);
                        }
                    }
                    const int bm = kb / p.kb_per_b;
                    if (GM > 1)   // every group reads all token tiles: keep them in L2 ahead of the weights
                        tma_load_2d_hint(b, &p.tb[bm], &full[stage], (kb - bm * p.kb_per_b) * 64, m_tile * NT, pol_b);
                    else
                        tma_load_2d(b, &p.tb[bm], &full[stage], (kb - bm * p.kb_per_b) * 64, m_tile * NT);
                    ++issued;
                    if (++stage == S) { stage = 0; ++round; }
                }
                u += kb1 - kb0;
            }
            if (*abort_flag) {
                // Let the copies already issued land before the CTA exits.
                long long first = issued > S ? issued - S : 0;
                for (long long i = first; i < issued; ++i) {
                    volatile int never = 0;
                    mbar_wait(&full[i % S], (uint32_t)((i / S) & 1), &never, nullptr);
                }
            }
        }
        // Finishing inputs of the last tile of a wide-tile CTA, issued by the whole warp
        // once the epilogue posts the plan: chunk c into buffer c % depth, once the
        // epilogue has consumed the chunk that buffer held.
        __syncwarp();
        if (NT >= 64 && u_begin < u_end && !*abort_flag && mbar_wait(land_go, 0, abort_flag, p.status)) {
            const LandPlan pl = *plan;
            if (pl.depth > 0) {
                fence_proxy_async_global();   // the partials, seen through the epilogue's acquire
                int nis = 0;
                for (int c = 0; c < pl.nchunks; ++c) {
                    if (c >= pl.depth) {
                        const bool fr = lane != 0 || mbar_wait(&lfree[c % pl.depth], (uint32_t)((c / pl.depth - 1) & 1),
                                                               abort_flag, p.status);
                        if (!__shfl_sync(0xffffffffu, (int)fr, 0)) break;
                    }
                    uint64_t* bar = &landc[c % pl.depth];
                    uint8_t* dst = smem + (size_t)(c % pl.depth) * pl.lbuf;
                    uint8_t* aux = dst + (size_t)pl.n_peer * (CH * 128 * 4);
                    // RoPE rows: one copy per run of consecutive positions of one request,
                    // issued by the lane of the run's first token
                    const void* rsrc = nullptr;
                    uint32_t rbytes = 0;
                    if (pl.aux == 2) {
                        const int tk = c * CH + lane;
                        const int b = lds_s32(tok_b_a + tk * 4u), pos = lds_s32(tok_pos_a + tk * 4u);
                        const int pb = __shfl_up_sync(0xffffffffu, b, 1), ppos = __shfl_up_sync(0xffffffffu, pos, 1);
                        const bool valid = b >= 0;
                        const bool start = valid && !(lane > 0 && pb == b && ppos + 1 == pos);
                        const uint32_t starts = __ballot_sync(0xffffffffu, start), valids = __ballot_sync(0xffffffffu, valid);
                        if (start) {
                            const uint32_t stops = (starts | ~valids) & ~((2u << lane) - 1u);   // lanes after this one that end the run
                            const int f = stops ? __ffs(stops) - 1 : 32;
                            rsrc = p.rope + (size_t)pos * (p.d >> 1);
                            rbytes = (uint32_t)((f - lane) * pl.aux_row);
                        }
                    }
                    const uint32_t total = __reduce_add_sync(0xffffffffu, rbytes) + (uint32_t)(pl.n_peer * CH * 128 * 4) +
                                           (pl.aux == 1 ? (uint32_t)(CH * 128 * 2) : 0u);
                    if (lane == 0) mbar_arrive_expect_tx(bar, total);
                    __syncwarp();
                    if (lane < pl.n_peer)
                        bulk_load(dst + (size_t)lane * (CH * 128 * 4), pl.psrc[lane] + (size_t)c * CH * 128,
                                  (uint32_t)(CH * 128 * 4), bar);
                    if (rbytes) bulk_load(aux + (size_t)lane * pl.aux_row, rsrc, rbytes, bar);
                    if (pl.aux == 1 && lane == 0) tma_load_2d(aux, &p.tx, bar, pl.tx_x, pl.tx_y0 + c * CH);
                    ++nis;
                }
                // every issued copy lands before the CTA can leave (the latest chunk of each buffer)
                if (lane == 0)
                    for (int b = 0; b < pl.depth && b < nis; ++b) {
                        const int last = b + pl.depth * ((nis - 1 - b) / pl.depth);
                        volatile int never = 0;
                        mbar_wait(&landc[b], (uint32_t)((last / pl.depth) & 1), &never, nullptr);
                    }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        griddep_wait();
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16_f32(128, NT);
            int stage = 0, seg = 0;
            uint32_t round = 0;
            bool ok = true;
            for (long long u = u_begin; u < u_end && ok;) {
                const int kb0 = (int)(u % KB);
                const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
                const int buf = seg & 1;
                const uint32_t use = (uint32_t)(seg >> 1);
                if (!mbar_wait(&acce[buf], (use & 1) ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(buf * NT);
                uint64_t* const landed = p.ssq_in ? ready : full;   // normalised by warp 6 first
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&landed[stage], round & 1, abort_flag, p.status)) { ok = false; break; }
                    if (trace && seg == 0 && kb == kb0) trace[2] = (long long)globaltimer_ns();
                    tc_fence_after();
                    const uint64_t ad = umma_desc_sw128(smem_u32(sA + stage * C::A_BYTES));
                    const uint64_t bd = umma_desc_sw128(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc_mma_bf16(d, ad + 2 * k, bd + 2 * k, IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
                    tc_commit(&empty[stage]);
                    if (++stage == S) { stage = 0; ++round; }
                }
                if (!ok) break;
                tc_commit(&accf[buf]);
                ++seg;
                u += kb1 - kb0;
            }
            if (trace) trace[3] = (long long)globaltimer_ns();
            if (*abort_flag) {
                // Drain the MMAs already issued before TMEM is released.
                tc_commit(drain);
                volatile int never = 0;
                mbar_wait(drain, 0, &never, nullptr);
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------------------ B normalisers (warps 6, 7)
        if (p.ssq_in) {
            const int nl = (warp - 6) * 32 + lane;   // 0..63 over the two warps
            float* inv_w = inv_s + (warp - 6) * NT;
            // The gain is a weight (independent of the previous kernel): stage it in
            // shared memory before the dependency wait, so no stage waits on a
            // global load of its slice.
            const bool gain_smem = p.K <= C::GAIN_MAX;
            if (gain_smem)
                for (int i = nl * 8; i < p.K; i += 64 * 8)
                    *reinterpret_cast<uint4*>(sgain + i) = __ldg(reinterpret_cast<const uint4*>(p.gain + i));
            named_bar_sync(2, 64);   // the staged gain; the only barrier between the two warps
            griddep_wait();
            int stage = 0, cur_mt = -1;
            uint32_t round = 0;
            bool ok = true;
            for (long long u = u_begin; u < u_end && ok;) {
                const long long t = tile_of(u);
                const int kb0 = (int)(u % KB);
                const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
                const int m_tile = (int)(t % m_tiles);
                // n-tile 0's k-blocks cover every feature once: its stages also go to norm_out
                const bool copy_out = p.norm_out && t / m_tiles == 0;
                if (m_tile != cur_mt) {
                    // inverse RMS of the m-tile's rows from the producer's per-tile
                    // partial sums; each warp keeps its own copy, so the two warps never
                    // wait for each other inside the stage loop.  A row's tiles are split
                    // into G contiguous runs, one per lane, each added in tile order from
                    // loads issued 16 at a time, then the G runs meet in a fixed butterfly:
                    // the same order in every CTA, and one or two round trips of latency
                    // instead of one per tile.
                    __syncwarp();
                    constexpr int G = NT < 32 ? 32 / NT : 1;   // lanes per row
                    const int T = p.ssq_tiles, per = (T + G - 1) / G;
                    for (int r0 = 0; r0 < NT; r0 += 32 / G) {
                        const int r = r0 + lane / G, g = lane % G;
                        const int m = m_tile * NT + r;
                        float ss = 0.f;
                        if (r < NT && m < p.M) {
                            const int j1 = min(T, (g + 1) * per);
                            for (int j = g * per; j < j1; j += 16) {
                                float part[16];
#pragma unroll
                                for (int k = 0; k < 16; ++k)
                                    part[k] = j + k < j1 ? __ldcg(p.ssq_in + (size_t)(j + k) * p.ssq_ld + m) : 0.f;
#pragma unroll
                                for (int k = 0; k < 16; ++k) ss += part[k];
                            }
                        }
#pragma unroll
                        for (int off = 1; off < G; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                        if (r < NT && g == 0) inv_w[r] = 1.0f / sqrtf(ss / (float)p.norm_h + p.eps);
                    }
                    __syncwarp();
                    cur_mt = m_tile;
                }
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&full[stage], round & 1, abort_flag, p.status)) { ok = false; break; }
                    // the stage's NT x 64 tile in the 128-byte swizzle: row r at r * 128 bytes,
                    // its 16-byte chunk j holds elements 8 (j ^ (r & 7)) .. + 7 of the k-block
                    uint8_t* bt = sB + stage * C::B_BYTES;
#pragma unroll 2
                    for (int ch = nl; ch < NT * 8; ch += 64) {
                        const int r = ch >> 3, j = ch & 7;
                        const int f0 = kb * 64 + 8 * (j ^ (r & 7));
                        uint4* ptr = reinterpret_cast<uint4*>(bt + r * 128 + j * 16);
                        const uint4 xv = *ptr;
                        const uint4 gv = gain_smem ? *reinterpret_cast<const uint4*>(sgain + f0)
                                                   : __ldg(reinterpret_cast<const uint4*>(p.gain + f0));
                        const __nv_bfloat16* xe = reinterpret_cast<const __nv_bfloat16*>(&xv);
                        const __nv_bfloat16* ge = reinterpret_cast<const __nv_bfloat16*>(&gv);
                        const float inv = inv_w[r];
                        uint4 out;
                        __nv_bfloat16* oe = reinterpret_cast<__nv_bfloat16*>(&out);
#pragma unroll
                        for (int k = 0; k < 8; ++k) oe[k] = f2bf(bf2f(xe[k]) * inv * bf2f(ge[k]));
                        *ptr = out;
                        const int m = m_tile * NT + r;
                        if (copy_out && m < p.M)
                            *reinterpret_cast<uint4*>(p.norm_out + (size_t)m * p.norm_out_ld + f0) = out;
                    }
                    fence_proxy_async();   // the MMA reads the stage through the async proxy
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ready[stage]);
                    if (++stage == S) { stage = 0; ++round; }
                }
                u += kb1 - kb0;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        griddep_wait();
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int row = q * 32 + lane;          // weight-tile row = TMEM lane
        const int e = threadIdx.x - 64;         // 0..127
        int seg = 0;
        int tok_mt = -1;                        // m-tile whose token map tok_b / tok_pos holds
        for (long long u = u_begin; u < u_end;) {
            const long long t = tile_of(u);
            const int kb0 = (int)(u % KB);
            const int kb1 = (int)min((long long)KB, kb0 + (u_end - u));
            const int n_tile = (int)(t / m_tiles), m_tile = (int)(t % m_tiles);
            const int buf = seg & 1;
            const uint32_t use = (uint32_t)(seg >> 1);
            // Everything the epilogue needs that does not depend on this tile's sums is
            // gathered while the tile still accumulates, so that the finishing path
            // after the last MMA holds as few dependent memory round trips as possible:
            // the per-token request / position map of the cache-writing epilogues ...
            if ((p.epi == EPI_QKV || p.epi == EPI_INJECT) && m_tile != tok_mt) {
                named_bar_sync(1, 128);   // the previous tile's readers of the map are done
                if (p.epi == EPI_QKV) {
                    for (int te = e; te < NT; te += 128) {   // NT may exceed the 128 epilogue threads
                        const int m = m_tile * NT + te;
                        int b = -1, pos = -1;
                        if (m < p.M) {
                            const int bb = m / p.gamma;
                            if (p.req_ok[bb]) { b = bb; pos = p.len[bb] + (m - bb * p.gamma); }
                        }
                        if (pos < 0 || pos >= p.cap) b = -1;   // never write outside the request's slab
                        tok_b[te] = b;
                        tok_pos[te] = pos;
                    }
                } else {
                    // one thread per request marks the rows it owns in this m-tile
                    for (int te = e; te < NT; te += 128) tok_b[te] = -1;
                    named_bar_sync(1, 128);
                    const int m0 = p.row0 + m_tile * NT;   // global row of the tile's first column
                    for (int bb = e; bb < p.batch; bb += 128) {
                        const int rs = p.row_start[bb], rc = p.row_count[bb], L0 = p.len[bb];
                        if (rc <= 0 || L0 < 0 || L0 + rc > p.cap) continue;
                        const int lo = max(rs, m0), hi = min(min(rs + rc, m0 + NT), p.row0 + p.M);
                        for (int m = lo; m < hi; ++m) {
                            tok_b[m - m0] = bb;
                            tok_pos[m - m0] = L0 + (m - rs);
                        }
                    }
                }
                named_bar_sync(1, 128);
                tok_mt = m_tile;
            }
            // ... the weight-row -> output-feature mapping of this tile ...
            int mi = 0;
            if (!p.swiglu)
                while (mi + 1 < p.n_amat && n_tile >= p.amat[mi + 1].tile0) ++mi;
            const int lr = p.swiglu ? 0 : (n_tile - p.amat[mi].tile0) * 128 + row;
            const bool row_ok = p.swiglu ? true : (lr < p.amat[mi].rows);
            // ... and, for single-chunk tiles, the residual rows or the RoPE cos/sin
            // of the thread's output feature (only a finisher uses them).
            constexpr bool PRE = NT <= 16;
            float pre_x[PRE ? CH : 1];
            float2 pre_cs[PRE ? CH : 1];
            if constexpr (PRE) {
                if (p.epi == EPI_RESID) {
                    const __nv_bfloat16* o = (const __nv_bfloat16*)p.out;
#pragma unroll
                    for (int i = 0; i < CH; ++i) {
                        const int m = m_tile * NT + i;
                        pre_x[i] = (row_ok && m < p.M) ? bf2f(o[(size_t)m * p.ldo + lr]) : 0.f;
                    }
                } else if (p.epi == EPI_QKV || p.epi == EPI_INJECT) {
                    // rotated sections: q and k of the QKV GEMM (matrices 0, 1), K of each layer in
                    // the injection GEMM (even matrices); the same rule as the epilogue's `rotate`
                    const bool rot = p.epi == EPI_QKV ? mi <= 1 : (mi & 1) == 0;
                    const int half = p.d >> 1, ih = (lr % p.d) % half;
#pragma unroll
                    for (int i = 0; i < CH; ++i)
                        pre_cs[i] = (rot && row_ok && lds_s32(tok_b_a + i * 4u) >= 0)
                                        ? __ldg(&p.rope[(size_t)lds_s32(tok_pos_a + i * 4u) * half + ih])
                                                                     : make_float2(1.f, 0.f);
                }
            }
            // Split tiles.  By default a split tile is finished by its first
            // contributor, the CTA holding the tile's k-blocks from 0: its range ends
            // inside the tile, so the tile is its last segment, while every other
            // contributor's range starts inside the tile, so each publishes its partial
            // in its first segment and never waits on another CTA (no cycle of waits;
            // the grid is at most one CTA per SM, so all CTAs become resident).  The
            // finisher stores no partial of its own: one thread waits for the count of
            // published partials, before the accumulator wait so that the round trip
            // overlaps the CTA's last MMAs.  With p.last_arriver every contributor
            // publishes and counts, and the one that counts last finishes.
            // In cluster mode the peers' partials arrive in this CTA's shared memory
            // (distributed shared-memory stores completing on landb), so the finisher
            // waits on its own barrier; whole-grid mode counts published partials in
            // global memory.
            const bool whole = (kb0 == 0 && kb1 == KB);
            const bool fin_first = !whole && (CL || !p.last_arriver) && kb0 == 0;
            // contributors: partition indices firsti .. firsti + nc - 1 (CTAs cta_of(i));
            // tn: the tile's weight-tile index in partition units (its k-block 0 at tn * KB)
            const long long tn = GM > 1 ? t / m_tiles : t;
            int first = cta, firsti = rloc, nc = 1;
            if (!whole) {
                const uint32_t t32 = (uint32_t)(tn * KB - ubase), K32 = (uint32_t)KB, U32 = (uint32_t)Uloc,
                               P32 = (uint32_t)Ploc;
                if (WT) {
                    firsti = (int)skw32_owner(t32, U32, P32, wL, wd);
                    nc = (int)skw32_owner(t32 + K32 - 1, U32, P32, wL, wd) - firsti + 1;
                } else {
                    firsti = (int)sk32_owner(t32, U32, P32);
                    nc = (int)sk32_owner(t32 + K32 - 1, U32, P32) - firsti + 1;
                }
                first = cta_of(firsti);
            }
            // partial slot of the CTA with partition index i for this tile: its first
            // segment (slot 2 * CTA) or its last (2 * CTA + 1)
            // (32-bit arithmetic: the launcher keeps every unit index below 2^32)
            auto slot_of = [&](int i) -> int {
                const uint32_t b0 = WT ? skw32_begin((uint32_t)i, (uint32_t)Uloc, (uint32_t)Ploc, wL, wd)
                                       : sk32_begin((uint32_t)i, (uint32_t)Uloc, (uint32_t)Ploc);
                const uint32_t first_tn = ((uint32_t)ubase + b0) / (uint32_t)KB;
                return 2 * cta_of(i) + (first_tn == (uint32_t)tn ? 0 : 1);
            };
            bool ok = true;
            if (fin_first) {
                if (CL)
                    ok = mbar_wait(landb, 0, abort_flag, p.status);
                else if (e == 0)
                    ok = count_wait(&p.counters[t], nc - 1, abort_flag, p.status);
            }
            ok = ok && mbar_wait(&accf[buf], use & 1, abort_flag, p.status);
            if (named_bar_or(1, 128, !ok)) break;   // leave together: later named barriers stay matched
            if (trace && e == 0) trace[4] = (long long)globaltimer_ns();
            tc_fence_after();
            const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * NT);
            // Whole-grid finisher: the tile is its last segment, so once its accumulator
            // is ready its ring is idle (every stage consumed, no load in flight): the
            // peers' partials land there in one round trip of bulk copies instead of
            // rounds of register loads.
            const bool land_ring =
                NT <= 32 && fin_first && !CL && nc > 1 && (nc - 1) * NT * 512 <= S * C::A_BYTES;
            if (land_ring) {
                if (e == 0) {
                    fence_proxy_async_global();   // the partials seen through the count's acquire
                    mbar_arrive_expect_tx(landb, (uint32_t)((nc - 1) * NT * 512));
                    for (int b = 1; b < nc; ++b)
                        bulk_load(sA + (size_t)(b - 1) * NT * 512, p.partial + (size_t)slot_of(firsti + b) * NT * 128,
                                  (uint32_t)(NT * 512), landb);
                }
                const bool lok = mbar_wait(landb, 0, abort_flag, p.status);
                if (!lok && e == 0) {
                    volatile int never = 0;   // let the copies land before the CTA can leave
                    mbar_wait(landb, 0, &never, nullptr);
                }
                if (named_bar_or(1, 128, !lok)) break;
            }
            // Wider tiles (NT >= 64) finished in the CTA's last segment: the ring is idle
            // then (every stage consumed, no load in flight), so what each CH-token chunk
            // of the epilogue reads from global memory lands there by bulk copies, up to
            // three chunks ahead of the chunk being finished, instead of every chunk
            // waiting on rounds of dependent register loads: the peers' partials (the CH
            // columns of a chunk are contiguous in a column-major partial) and the
            // epilogue's inputs, the residual rows of the chunk's tokens (EPI_RESID) or
            // their RoPE rows (rotated sections of EPI_QKV / EPI_INJECT).
            static_assert(NT < 64 || CH == 32, "32-token chunks");
            constexpr int LC_BYTES = CH * 128 * 4;          // one chunk of one partial
            constexpr int RING_BYTES = S * C::STAGE_BYTES;
            const bool rot_tile = p.epi == EPI_QKV ? mi <= 1 : (p.epi == EPI_INJECT && (mi & 1) == 0);
            const int n_peer = fin_first ? nc - 1 : 0;
            const int aux_row = p.epi == EPI_RESID ? (p.has_tx ? 128 * 2 : -1)
                                                   : (rot_tile ? (p.d >> 1) * 8 : 0);   // bytes per token
            const int lbuf = n_peer * LC_BYTES + CH * max(aux_row, 0);                            // bytes per chunk
            const bool last_seg = u + (kb1 - kb0) == u_end;
            const int lc_depth = (NT >= 64 && !CL && last_seg && (fin_first || whole) && aux_row >= 0 && lbuf > 0 &&
                                  lbuf <= RING_BYTES)
                                     ? min(3, min(NT / CH, RING_BYTES / lbuf))
                                     : 0;
            const int lcd = lc_depth > 0 ? lc_depth : 1;   // buffers (a divisor when the mode is off)
            if (NT >= 64 && last_seg) {
                // Post the landing plan to the producer warp (every CTA, once, at its last
                // segment; depth 0 when nothing lands).
                if (e < 32) {
                    if (lc_depth > 0 && e < n_peer) plan->psrc[e] = p.partial + (size_t)slot_of(firsti + 1 + e) * NT * 128;
                    __syncwarp();
                    if (e == 0) {
                        plan->depth = lc_depth;
                        plan->nchunks = NT / CH;
                        plan->lbuf = lbuf;
                        plan->n_peer = n_peer;
                        plan->aux = p.epi == EPI_RESID ? 1 : (rot_tile ? 2 : 0);
                        plan->aux_row = max(aux_row, 0);
                        plan->tx_x = (n_tile - p.amat[mi].tile0) * 128;
                        plan->tx_y0 = m_tile * NT;
                        mbar_arrive(land_go);
                    }
                }
            }
            bool lost = false;
            bool finish = true;
            if (!whole && !fin_first && CL) {
                // Send the partial (all NT columns of this thread's row) into the
                // finisher's landing slot for this rank, 16 bytes per store.
                const uint32_t fr = (uint32_t)(first - cbase);
                const uint32_t slot = (uint32_t)(rloc - (first - cbase) - 1);
                const uint32_t raddr = mapa_shared(smem_u32(land + ((size_t)slot * 128 + row) * C::LAND_LD), fr);
                const uint32_t rbar = mapa_shared(smem_u32(landb), fr);
#pragma unroll 1
                for (int c0 = 0; c0 < NT; c0 += 16) {
                    float v[16];
                    tmem_ld16(tb + c0, v);
#pragma unroll
                    for (int i = 0; i < 16; i += 4)
                        st_async_v4(raddr + (uint32_t)(c0 + i) * 4, v[i], v[i + 1], v[i + 2], v[i + 3], rbar);
                }
                finish = false;
            } else if (!whole && !fin_first) {
                float* dst = p.partial + (size_t)slot_of(rloc) * NT * 128;
#pragma unroll 1
                for (int c0 = 0; c0 < NT; c0 += 16) {
                    float v[16];
                    tmem_ld16(tb + c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) __stcg(dst + (c0 + i) * 128 + row, v[i]);
                }
                // Release the CTA's partial and count it: the barrier orders every
                // thread's stores before one thread's gpu-scope fence and atomic; the
                // finisher's acquire (a fence after the atomic for the last arriver)
                // and the barrier after it make the partials visible to all its threads.
                named_bar_sync(1, 128);
                if (p.last_arriver) {
                    if (e == 0) {
                        __threadfence();
                        const int old = atomicAdd(&p.counters[t], 1);
                        const bool last = old == nc - 1;
                        if (last) __threadfence();
                        *s_flag = last ? 1 : 0;
                    }
                    named_bar_sync(1, 128);
                    finish = (lds_s32(smem_u32(s_flag)) != 0);
                } else {
                    if (e == 0) {
                        __threadfence();
                        atomicAdd(&p.counters[t], 1);
                    }
                    finish = false;
                }
            }
            if (finish) {
#pragma unroll 1
                for (int c0 = 0; c0 < NT; c0 += CH) {
                    float v[CH];
#pragma unroll
                    for (int h = 0; h < CH; h += 16) tmem_ld16(tb + c0 + h, v + h);
                    if (lc_depth > 0) {
                        // this CTA first (the first contributor), then the landed chunks of
                        // the partials in contributor order
                        const int ci = c0 / CH;
                        const bool lok = mbar_wait(&landc[ci % lcd], (uint32_t)((ci / lcd) & 1), abort_flag, p.status);
                        if (named_bar_or(1, 128, !lok)) {   // the producer lets its copies land
                            lost = true;
                            break;
                        }
                        if (n_peer > 0) {
                            uint32_t src = smem_u32(smem + (size_t)(ci % lcd) * lbuf) + (uint32_t)row * 4u;
                            float acc[CH];
#pragma unroll
                            for (int i = 0; i < CH; ++i) acc[i] = 0.0f + v[i];
                            for (int b = 0; b < n_peer; ++b, src += CH * 128 * 4) {
#pragma unroll
                                for (int i = 0; i < CH; ++i) acc[i] += lds_f32(src + i * 512u);
                            }
#pragma unroll
                            for (int i = 0; i < CH; ++i) v[i] = acc[i];
                        }
                    } else if (!whole && CL) {
                        // this CTA first, then the peers' partials in rank order
                        float acc[CH];
#pragma unroll
                        for (int i = 0; i < CH; ++i) acc[i] = 0.0f + v[i];
                        for (int b = 1; b < nc; ++b) {
                            const uint32_t src = smem_u32(land + ((size_t)(b - 1) * 128 + row) * C::LAND_LD + c0);
#pragma unroll
                            for (int i = 0; i < CH; i += 4) {
                                const float4 w = lds_f32x4(src + i * 4u);
                                acc[i] += w.x;
                                acc[i + 1] += w.y;
                                acc[i + 2] += w.z;
                                acc[i + 3] += w.w;
                            }
                        }
#pragma unroll
                        for (int i = 0; i < CH; ++i) v[i] = acc[i];
                    } else if (!whole && land_ring) {
                        // this CTA first (it is the first contributor), then the landed
                        // partials in contributor order
                        float acc[CH];
#pragma unroll
                        for (int i = 0; i < CH; ++i) acc[i] = 0.0f + v[i];
                        for (int b = 1; b < nc; ++b) {
                            const uint32_t src = smem_u32(sA) + (uint32_t)(((b - 1) * NT * 128 + c0 * 128 + row) * 4);
#pragma unroll
                            for (int i = 0; i < CH; ++i) acc[i] += lds_f32(src + i * 512u);
                        }
#pragma unroll
                        for (int i = 0; i < CH; ++i) v[i] = acc[i];
                    } else if (!whole) {
                        float acc[CH];
#pragma unroll
                        for (int i = 0; i < CH; ++i) acc[i] = 0.0f;
                        constexpr int MAXB = CH <= 16 ? 4 : 2;
                        for (int b0 = 0; b0 < nc; b0 += MAXB) {
                            float pv[MAXB][CH];
#pragma unroll
                            for (int bi = 0; bi < MAXB; ++bi) {
                                const int pi = firsti + b0 + bi;
                                if (b0 + bi < nc && pi != rloc) {
                                    const float* src = p.partial + (size_t)slot_of(pi) * NT * 128;
#pragma unroll
                                    for (int i = 0; i < CH; ++i) pv[bi][i] = __ldcg(src + (c0 + i) * 128 + row);
                                }
                            }
#pragma unroll
                            for (int bi = 0; bi < MAXB; ++bi) {
                                if (b0 + bi < nc) {
                                    const bool own = firsti + b0 + bi == rloc;
#pragma unroll
                                    for (int i = 0; i < CH; ++i) acc[i] += own ? v[i] : pv[bi][i];
                                }
                            }
                        }
#pragma unroll
                        for (int i = 0; i < CH; ++i) v[i] = acc[i];
                    }
                    // ---------------------------------------------- epilogues
                    const int mbase = m_tile * NT + c0;
                    switch (p.epi) {
                    case EPI_F32: {
                        float* o = (float*)p.out;
                        if (row_ok)
#pragma unroll
                            for (int i = 0; i < CH; ++i)
                                if (mbase + i < p.M) o[(size_t)(mbase + i) * p.ldo + lr] = v[i];
                        break;
                    }
                    case EPI_BF16:
                    case EPI_RESID: {
                        // The rounded outputs go through shared memory token-major, so
                        // that they leave in 16-byte stores and each token's sum of
                        // squares over the tile's features is one short butterfly.
                        __nv_bfloat16* o = (__nv_bfloat16*)p.out;
                        if (p.epi == EPI_RESID) {
                            float rv[CH];
                            if constexpr (PRE) {
#pragma unroll
                                for (int i = 0; i < CH; ++i) rv[i] = pre_x[i];
                            } else if (lc_depth > 0) {
                                // the chunk's residual rows landed after the partials
                                const uint32_t xs = smem_u32(smem + (size_t)((c0 / CH) % lcd) * lbuf + (size_t)n_peer * LC_BYTES) +
                                                    (uint32_t)row * 2u;
                                // loaded unconditionally (the landed rows always exist), then
                                // selected: a load under a condition serialises the chunk
#pragma unroll
                                for (int i = 0; i < CH; ++i) {
                                    const float xv = lds_bf16_as_f32(xs + i * 256u);
                                    rv[i] = (row_ok && mbase + i < p.M) ? xv : 0.f;
                                }
                            } else {
#pragma unroll
                                for (int i = 0; i < CH; ++i)
                                    rv[i] = (row_ok && mbase + i < p.M) ? bf2f(o[(size_t)(mbase + i) * p.ldo + lr]) : 0.f;
                            }
#pragma unroll
                            for (int i = 0; i < CH; ++i) xout[i * 128 + row] = f2bf(rv[i] + v[i]);
                        } else {
#pragma unroll
                            for (int i = 0; i < CH; ++i) xout[i * 128 + row] = f2bf(v[i]);
                        }
                        named_bar_sync(1, 128);
                        const int nrows = p.amat[mi].rows, rbase = (n_tile - p.amat[mi].tile0) * 128;
#pragma unroll
                        for (int k = 0; k < CH / 8; ++k) {
                            const int c = e + 128 * k, i = c >> 4, r0 = (c & 15) * 8;
                            const int m = mbase + i, f = rbase + r0;
                            const bool in = m < p.M && f < nrows;   // rows come in multiples of 8
                            const uint4 w = lds_u32x4(xch_a + (uint32_t)(i * 128 + r0) * 2u);
                            if (in) *(uint4*)(o + (size_t)m * p.ldo + f) = w;
                            if (p.ssq_out) {
                                // the 8 features in order, then the 16 pieces of the token
                                // in a fixed butterfly
                                float sq = 0.f;
                                if (in) {
                                    const __nv_bfloat16* b8 = (const __nv_bfloat16*)&w;
#pragma unroll
                                    for (int j = 0; j < 8; ++j) {
                                        const float xf = bf2f(b8[j]);
                                        sq = fmaf(xf, xf, sq);
                                    }
                                }
#pragma unroll
                                for (int off = 8; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
                                if ((c & 15) == 0 && m < p.M) p.ssq_out[(size_t)n_tile * p.ssq_ld + m] = sq;
                            }
                        }
                        named_bar_sync(1, 128);
                        break;
                    }
                    case EPI_SWIGLU: {
                        // Rows 0..63 of the tile are gate rows, 64..127 the matching up
                        // rows.  Both cross through the exchange buffer, so that all four
                        // warps form products: thread e takes gate row e % 64 and half of
                        // the chunk's tokens; the bf16 products then go through the buffer's
                        // lower rows once every thread has read its pairs.
#pragma unroll
                        for (int i = 0; i < CH; ++i) xch[row * (CH + 1) + i] = v[i];
                        named_bar_sync(1, 128);
                        const int g = e & 63, i0 = (e >> 6) * (CH / 2);
                        float prod[CH / 2];
#pragma unroll
                        for (int j = 0; j < CH / 2; ++j) {
                            const float gv = lds_f32(xch_a + (uint32_t)(g * (CH + 1) + i0 + j) * 4u);
                            const float uv = lds_f32(xch_a + (uint32_t)((g + 64) * (CH + 1) + i0 + j) * 4u);
                            prod[j] = silu(gv) * uv;
                        }
                        named_bar_sync(1, 128);
#pragma unroll
                        for (int j = 0; j < CH / 2; ++j) xout[(i0 + j) * 64 + g] = f2bf(prod[j]);
                        named_bar_sync(1, 128);
                        __nv_bfloat16* o = (__nv_bfloat16*)p.out;
#pragma unroll
                        for (int k = 0; k < CH / 16; ++k) {
                            const int c = e + 128 * k, i = c >> 3, r0 = (c & 7) * 8;
                            const int m = mbase + i;
                            if (m < p.M)
                                *(uint4*)(o + (size_t)m * p.ldo + n_tile * 64 + r0) = lds_u32x4(xch_a + (uint32_t)(i * 64 + r0) * 2u);
                        }
                        named_bar_sync(1, 128);
                        break;
                    }
                    case EPI_QKV:
                    case EPI_INJECT: {
                        // Section of this weight matrix: QKV -> 0 q, 1 k, 2 v;
                        // inject -> (layer, kind) = (mi / 2, mi % 2).
                        const bool is_q = (p.epi == EPI_QKV && mi == 0);
                        const int kind = (p.epi == EPI_QKV) ? mi - 1 : (mi & 1);
                        const int layer = (p.epi == EPI_QKV) ? p.layer : p.layer + (mi >> 1);
                        const bool rotate = is_q || kind == 0;
                        const int d = p.d, half = d >> 1;
                        const int i_in = lr % d;
#pragma unroll
                        for (int i = 0; i < CH; ++i) xch[row * (CH + 1) + i] = v[i];
                        named_bar_sync(1, 128);
                        // rotate-half RoPE of every column (the partner feature of the same
                        // head from the exchange buffer), rounded to bf16 in registers
                        const int prow = (i_in < half) ? row + half : row - half;
                        float2 cs[CH];
                        if constexpr (PRE) {
#pragma unroll
                            for (int i = 0; i < CH; ++i) cs[i] = pre_cs[i];
                        } else if (lc_depth > 0 && rotate) {
                            // the chunk's RoPE rows landed after the partials
                            const uint32_t rs = smem_u32(smem + (size_t)((c0 / CH) % lcd) * lbuf + (size_t)n_peer * LC_BYTES) +
                                                (uint32_t)(i_in % half) * 8u;
#pragma unroll
                            for (int i = 0; i < CH; ++i) {
                                const int b = lds_s32(tok_b_a + (c0 + i) * 4u);
                                const float2 r = lds_f32x2(rs + (uint32_t)(i * half) * 8u);   // unconditional, then selected
                                cs[i] = (row_ok && b >= 0) ? r : make_float2(1.f, 0.f);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < CH; ++i) {
                                const int b = lds_s32(tok_b_a + (c0 + i) * 4u);
                                cs[i] = (rotate && row_ok && b >= 0)
                                            ? __ldg(&p.rope[(size_t)lds_s32(tok_pos_a + (c0 + i) * 4u) * half + (i_in % half)])
                                            : make_float2(1.f, 0.f);
                            }
                        }
                        __nv_bfloat16 y[CH];
#pragma unroll
                        for (int i = 0; i < CH; ++i) {
                            float x = v[i];
                            const float pr = lds_f32(xch_a + (uint32_t)(prow * (CH + 1) + i) * 4u);   // unconditional
                            if (rotate) x = (i_in < half) ? (x * cs[i].x - pr * cs[i].y) : (x * cs[i].x + pr * cs[i].y);
                            y[i] = f2bf(x);
                        }
                        named_bar_sync(1, 128);
#pragma unroll
                        for (int i = 0; i < CH; ++i) xout[i * 128 + row] = y[i];
                        named_bar_sync(1, 128);
                        // 8 features of one token per 16-byte store: a q row, or a K/V cache
                        // row of the token's request and position
                        const int nrows = p.amat[mi].rows, rbase = (n_tile - p.amat[mi].tile0) * 128;
#pragma unroll
                        for (int k = 0; k < CH / 8; ++k) {
                            const int c = e + 128 * k, i = c >> 4, r0 = (c & 15) * 8;
                            const int b = lds_s32(tok_b_a + (c0 + i) * 4u), f = rbase + r0;
                            const int tpos = lds_s32(tok_pos_a + (c0 + i) * 4u);
                            const uint4 w = lds_u32x4(xch_a + (uint32_t)(i * 128 + r0) * 2u);
                            if (b >= 0 && f < nrows) {
                                __nv_bfloat16* dst =
                                    is_q ? (__nv_bfloat16*)p.out + (size_t)(mbase + i) * p.ldo + f
                                         : p.slab + (size_t)b * p.s_req + (size_t)layer * p.s_layer +
                                               (size_t)kind * p.s_kind + (size_t)(f / d) * p.s_kv +
                                               (size_t)tpos * d + (f % d);
                                *(uint4*)dst = w;
                            }
                        }
                        named_bar_sync(1, 128);
                        break;
                    }
                    case EPI_LMHEAD: {
                        // Optional logits (the drafting rows only), then the top-2 of each
                        // token column over the tile's 128 vocabulary rows: the columns
                        // cross shared memory, G = 128 / CH threads scan CH rows each in
                        // row order, and a butterfly over the G threads merges them (ties
                        // of the top value go to the lower id, whatever the order).
                        const int vid = lr;   // vocab id (lm_head is one matrix)
                        if (p.logits && row_ok) {
#pragma unroll 1
                            for (int i = 0; i < CH; ++i) {
                                const int m = mbase + i;
                                if (m >= p.M) break;
                                int lrow = m;
                                if (p.lm_gamma) {
                                    const int j = m % p.lm_gamma;
                                    lrow = j == 0 ? -1 : (m / p.lm_gamma) * (p.lm_gamma - 1) + j - 1;
                                }
                                if (lrow >= 0) p.logits[(size_t)lrow * p.vocab + vid] = v[i];
                            }
                        }
#pragma unroll
                        for (int i = 0; i < CH; ++i) xch[row * (CH + 1) + i] = row_ok ? v[i] : -INFINITY;
                        named_bar_sync(1, 128);
                        constexpr int G = 128 / CH;
                        const int i = e / G, j = e % G, vbase = n_tile * 128;
                        float a1 = -INFINITY, a2 = -INFINITY;
                        int ai = 0x7fffffff;
#pragma unroll
                        for (int k = 0; k < CH; ++k) {
                            const int r = j + G * k;
                            top2_merge(a1, ai, a2, lds_f32(xch_a + (uint32_t)(r * (CH + 1) + i) * 4u), vbase + r, -INFINITY);
                        }
#pragma unroll
                        for (int off = G / 2; off > 0; off >>= 1) {
                            const float b1 = __shfl_xor_sync(0xffffffffu, a1, off);
                            const int bi = __shfl_xor_sync(0xffffffffu, ai, off);
                            const float b2 = __shfl_xor_sync(0xffffffffu, a2, off);
                            top2_merge(a1, ai, a2, b1, bi, b2);
                        }
                        if (j == 0 && mbase + i < p.M)
                            p.records[(size_t)(mbase + i) * p.n_tiles + n_tile] = make_float4(a1, __int_as_float(ai), a2, 0.0f);
                        named_bar_sync(1, 128);
                        break;
                    }
                    default:
                        break;
                    }
                    // the chunk's buffer is free for the chunk lc_depth ahead once every
                    // thread is done with it
                    if (lc_depth > 0) mbar_arrive(&lfree[(c0 / CH) % lcd]);
                }
                if (lost) break;
                if (!whole && !CL && e == 0) p.counters[t] = 0;
            }
            tc_fence_before();
            mbar_arrive(&acce[buf]);
            ++seg;
            u += kb1 - kb0;
        }
        if (trace && e == 0) trace[5] = (long long)globaltimer_ns();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (CL) {
        // no CTA leaves while a peer may still store into its shared memory
        cluster_arrive();
        cluster_wait();
    }
    if (trace && threadIdx.x == 0) {
        trace[6] = (long long)globaltimer_ns();
        trace[7] = clock64() - clk0;
    }
}

template <int NT, bool CLU>
static cudaError_t set_smem_attr() {
    static bool done = false;
    if (done) return cudaSuccess;
    cudaError_t e =
        cudaFuncSetAttribute(k_gemm_tc<NT, CLU>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<NT, CLU>::SMEM);
    done = e == cudaSuccess;
    return e;
}

template <int NT, bool CLU>
static int launch_nt(GemmParams& p, cudaStream_t stream) {
    using C = GemmCfg<NT, CLU>;
    cudaError_t e = set_smem_attr<NT, CLU>();
    if (e != cudaSuccess) return (int)e;
    if (CLU) {
        ensure_carveout((const void*)k_gemm_tc<NT, CLU>);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(p.ctas);
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = (size_t)C::SMEM;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)p.cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, k_gemm_tc<NT, CLU>, p);
    } else {
        e = launch_k(k_gemm_tc<NT, CLU>, dim3(p.ctas), dim3(C::THREADS), (size_t)C::SMEM, stream, p);
    }
    if (e != cudaSuccess) return (int)e;
    return (int)cudaGetLastError();
}

// Clusters of c CTAs of the 16-token kernel that can be resident at once (the
// clusters of one launch must fit a GPC each), cached; 0 if none.
static int max_active_clusters16(int c) {
    static int cached[9] = {-1, -1, -1, -1, -1, -1, -1, -1, -1};
    if (c < 2 || c > 8) return 0;
    if (cached[c] >= 0) return cached[c];
    int n = 0;
    if (set_smem_attr<16, true>() == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(c * 8);
        cfg.blockDim = dim3(GemmCfg<16, true>::THREADS);
        cfg.dynamicSmemBytes = (size_t)GemmCfg<16, true>::SMEM;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)c;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, (const void*)k_gemm_tc<16, true>, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    cached[c] = n;
    return n;
}

// Cluster mode pays when the cluster partition's longest CTA range (whole tiles per
// cluster, split over its CTAs) is shorter than the whole-grid range plus the
// global-memory split-tile fix-up, which costs about kFixupUnits weight tiles of
// streaming at the end of every launch.  Off by default: on a 148-SM B200, 74 / 45 /
// 33 clusters of 2 / 3 / 4 CTAs are resident, which fits none of the 16-token
// projections of the drafters here well enough (QKV's 48 tiles need 48 clusters of
// 3; the O-projection's 32 tiles on 128 CTAs with the shallower ring measured
// slower than the whole-grid kernel).
constexpr long long kFixupUnits = 6;
static int g_max_cluster = 0;
int gemm_max_cluster() { return g_max_cluster; }
void set_gemm_max_cluster(int c) {
    constexpr int cmax = GemmCfg<16, true>::LAND_SLOTS + 1;
    g_max_cluster = c < 0 ? 0 : (c > cmax ? cmax : c);
}
int gemm_max_active_clusters(int c) { return max_active_clusters16(c); }

static void pick_cluster(GemmParams& p, int num_sms) {
    p.cluster = 0;
    if (g_max_cluster < 2 || p.whole_tiles) return;
    const long long T = (long long)p.n_tiles * p.m_tiles, KB = p.KB;
    long long best = (T * KB + num_sms - 1) / num_sms + kFixupUnits;
    for (int c = 2; c <= g_max_cluster; ++c) {
        if (KB < c) break;
        const long long Q = std::min<long long>(max_active_clusters16(c), std::min<long long>(T, num_sms / c));
        if (Q < 1) continue;
        const long long cost = (((T + Q - 1) / Q) * KB + c - 1) / c;
        if (cost < best) {
            best = cost;
            p.cluster = c;
            p.ctas = (int)(Q * c);
        }
    }
}

static int g_l2_prefetch = 0;
static int g_pre_stages = 6;   // measured: 6 of the ring's stages before the wait beat the whole ring
static int g_last_arriver = 0;
int gemm_pre_stages() { return g_pre_stages; }
void set_gemm_pre_stages(int stages) { g_pre_stages = stages < 0 ? 0 : stages; }
int gemm_last_arriver() { return g_last_arriver; }
void set_gemm_last_arriver(int on) { g_last_arriver = on != 0; }
int gemm_l2_prefetch() { return g_l2_prefetch; }
void set_gemm_l2_prefetch(int tiles) { g_l2_prefetch = tiles < 0 ? 0 : (tiles > 256 ? 256 : tiles); }

int launch_gemm_tc(GemmParams& p, int nt, int num_sms, cudaStream_t stream) {
    p.KB = (p.K + 63) / 64;
    p.m_tiles = (p.M + nt - 1) / nt;
    if (p.swiglu) {
        // n_tiles set by the caller (I / 64)
    } else {
        int nt_total = 0;
        for (int i = 0; i < p.n_amat; ++i) {
            p.amat[i].tile0 = nt_total;
            p.amat[i].ntiles = (p.amat[i].rows + 127) / 128;
            nt_total += p.amat[i].ntiles;
        }
        p.n_tiles = nt_total;
    }
    // The bf16 epilogues write 8 features of a token per 16-byte store: output rows,
    // row strides and K/V cache strides must keep 8-element pieces 16-byte aligned.
    if (p.epi != EPI_F32 && p.epi != EPI_LMHEAD) {
        const bool q_out = p.epi != EPI_INJECT;
        if (q_out && (((uintptr_t)p.out & 15) != 0 || p.ldo % 8 != 0)) return (int)cudaErrorInvalidValue;
        for (int i = 0; i < p.n_amat; ++i)
            if (p.amat[i].rows % 8 != 0) return (int)cudaErrorInvalidValue;
        if ((p.epi == EPI_QKV || p.epi == EPI_INJECT) &&
            (((uintptr_t)p.slab & 15) != 0 || p.d % 8 != 0 || p.s_req % 8 != 0 || p.s_layer % 8 != 0 ||
             p.s_kind % 8 != 0 || p.s_kv % 8 != 0))
            return (int)cudaErrorInvalidValue;
    }
    // Residual rows for the chunked landing of wide tiles: 32 tokens x 128 features
    // per copy (the kernel falls back to register loads without it).
    p.has_tx = 0;
    if (p.epi == EPI_RESID && nt >= 64 && p.n_amat == 1)
        p.has_tx = encode_bf16_rows(&p.tx, p.out, (uint64_t)p.amat[0].rows, (uint64_t)p.M, (uint64_t)p.ldo, 128, 32) ? 1 : 0;
    p.units = (long long)p.n_tiles * p.m_tiles * p.KB;
    if (p.units * (long long)kGemmMaxGrid >= (1LL << 32)) return (int)cudaErrorInvalidValue;   // 32-bit partition arithmetic
    const bool auto_grid = p.ctas <= 0;
    if (p.ctas <= 0 || p.ctas > num_sms) p.ctas = num_sms;
    if ((long long)p.ctas > p.units) p.ctas = (int)p.units;
    if (p.whole_tiles && (long long)p.ctas > p.units / p.KB) p.ctas = (int)(p.units / p.KB);
    if (p.units == 0) return 0;
    p.cluster = 0;
    if (nt == 16 && auto_grid) pick_cluster(p, num_sms);
    // Weighted shares only on the whole grid, when every late CTA keeps a unit and the
    // 32-bit partition arithmetic holds.
    if (p.late_deficit > 0) {
        const long long L = p.late_from, d = p.late_deficit, P = p.ctas;
        const long long E = p.units + (P - L) * d;
        if (p.whole_tiles || p.cluster >= 2 || L <= 0 || L >= P || p.units - L * d < P || P * E >= (1LL << 32))
            p.late_deficit = 0;
    }
    // Several token tiles: groups of m_tiles CTAs, one per token tile, when that keeps
    // at least 90 % of the grid busy and every group has work (a unit; with whole
    // tiles, a weight tile).
    p.grouped = 0;
    if (nt == 256 && auto_grid && p.cluster < 2 && p.m_tiles > 1) {
        int G = p.ctas / p.m_tiles;
        if (p.whole_tiles && G > p.n_tiles) G = p.n_tiles;
        if (G >= 1 && (long long)G * p.m_tiles * 10 >= (long long)p.ctas * 9 &&
            (long long)p.n_tiles * p.KB >= G) {
            p.grouped = 1;
            p.ctas = G * p.m_tiles;
            p.late_deficit = 0;
        }
    }
    switch (nt) {
    case 16: return p.cluster >= 2 ? launch_nt<16, true>(p, stream) : launch_nt<16, false>(p, stream);
    case 32: return launch_nt<32, false>(p, stream);
    case 64: return launch_nt<64, false>(p, stream);
    case 128: return launch_nt<128, false>(p, stream);
    case 256: return launch_nt<256, false>(p, stream);
    default: return (int)cudaErrorInvalidValue;
    }
}

}  // namespace df
