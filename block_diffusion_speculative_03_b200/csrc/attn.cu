// Block attention of the draft step (bf16 storage), split over the key axis
// across the CTAs of one thread-block cluster.
//
// For request b and kv head g, the G*gamma query rows (G = query heads per kv
// head) attend to every cached row [0, len) plus the gamma block rows that the
// QKV epilogue wrote at [len, len+gamma): no mask.  The `splits` CTAs of a
// cluster (b, g) each take one key range: K/V tiles of 64 rows x d arrive by
// TMA (128-byte swizzle, no multicast) into a 3-stage ring; each warp owns 16
// query rows (and a share of every tile's keys when there are fewer than 64
// rows), computes S = Q K^T and O += P V with mma.sync m16n8k16 (bf16 in, fp32
// accumulate), and keeps the online-softmax row max / sum with quad shuffles.
// Each CTA leaves its partial (m, l, O) in its own shared memory; after a
// cluster barrier every CTA merges a slice of the rows by reading all partials
// through distributed shared memory, and writes the bf16 output.  No partial
// goes through global memory and no second kernel is needed.
#include <cooperative_groups.h>

#include "attn.cuh"

namespace cg = cooperative_groups;

namespace df {

// Byte offset of element (r, c) in a [64 rows][D] bf16 tile stored as D/64
// column blocks of [64 rows][128 B] with the 128-byte swizzle (16-byte chunk
// index XOR row % 8), which is the layout TMA writes.
DF_DEV uint32_t sw_off(int r, int c) {
    return (uint32_t)((c >> 6) * (64 * 128) + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

template <int D>
__global__ void __launch_bounds__(128) k_attn_cluster(const __grid_constant__ AttnParams p) {
    constexpr int TILE_BYTES = 64 * D * 2;
    constexpr int NDT = D / 8;     // n-tiles of the output
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + TILE_BYTES;                   // [stages]
    uint8_t* sV = sK + kAttnStages * TILE_BYTES;     // [stages]
    uint64_t* bars = (uint64_t*)(sV + kAttnStages * TILE_BYTES);
    // After the key loop the ring is reused: per-warp results, then the CTA's partial.
    float* mo = (float*)(smem + TILE_BYTES);         // [4 warps][16][D]
    float2* mml = (float2*)(mo + 4 * 16 * D);        // [4 warps][16] (m, l)
    float* po = (float*)(mml + 4 * 16);              // [64][D]  partial O of this CTA
    float2* pml = (float2*)(po + 64 * D);            // [64]     (m, l) of this CTA
    float* wts = (float*)(pml + 64);                 // [64][4]  in-CTA merge weights
    float* cm = wts + 64 * 4;                        // [64][splits] peers' row max
    float* cl = cm + 64 * kAttnMaxSplits;            // [64][splits] peers' row sum
    float* cw = cl + 64 * kAttnMaxSplits;            // [64][splits] normalised merge weights
    __shared__ int s_abort;

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int nsplit = p.splits;
    const int g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) tma_prefetch_desc(&p.tmap);
    griddep_wait();
    griddep_launch();

    const int R = p.G * p.gamma;
    const int rows_per = (R + nsplit - 1) / nsplit;
    const int r_lo = rank * rows_per, r_hi = min(R, r_lo + rows_per);
    if (!p.req_ok[b]) {   // skipped request: zero output rows, no cluster traffic
        for (int r = r_lo; r < r_hi; ++r) {
            const int j = r / p.G, hh = r % p.G;
            __nv_bfloat16* dst = p.out + ((size_t)(b * p.gamma + j) * p.nq + (size_t)(g * p.G + hh)) * D;
            for (int c = tid; c < D; c += 128) dst[c] = f2bf(0.f);
        }
        return;
    }
    const int n = p.len[b] + p.gamma;
    const int kv0 = rank * p.chunk;
    const int kv1 = min(n, kv0 + p.chunk);
    const int ntiles = kv1 > kv0 ? (kv1 - kv0 + 63) / 64 : 0;
    int RT = (R + 15) / 16;
    if (RT == 3) RT = 4;
    const int NKS = 4 / RT;
    const int rt = warp % RT, ks = warp / RT;
    const int W = 64 / NKS;         // keys of each tile handled by this warp
    const long long rowK = (long long)b * p.rows_req + (long long)p.layer * p.rows_layer + (long long)g * p.rows_kv;
    const long long rowV = rowK + p.rows_kind;

    if (tid == 0) {
        s_abort = 0;
        for (int i = 0; i < kAttnStages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        for (int it = 0; it < min(ntiles, kAttnStages); ++it) {
            mbar_arrive_expect_tx(&bars[it], 2 * TILE_BYTES);
            for (int h = 0; h < D / 64; ++h) {
                tma_load_2d(sK + it * TILE_BYTES + h * 8192, &p.tmap, &bars[it], h * 64, (int)(rowK + kv0 + it * 64));
                tma_load_2d(sV + it * TILE_BYTES + h * 8192, &p.tmap, &bars[it], h * 64, (int)(rowV + kv0 + it * 64));
            }
        }
    }
    // Q tile: row r = j*G + h  <->  block position j, query head g*G + h.
    for (int idx = tid; idx < 64 * (D / 8); idx += 128) {
        const int r = idx / (D / 8), c = (idx % (D / 8)) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < R) {
            const int j = r / p.G, hh = r % p.G;
            const __nv_bfloat16* src = p.q + ((size_t)(b * p.gamma + j) * p.nq + (size_t)(g * p.G + hh)) * D + c;
            v = *reinterpret_cast<const uint4*>(src);
        }
        *reinterpret_cast<uint4*>(sQ + sw_off(r, c)) = v;
    }
    __syncthreads();

    uint32_t qa[D / 16][4];
    {
        const int mi = lane >> 3;
        const int r = rt * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int c = kk * 16 + (mi >> 1) * 8;
            ldmatrix_x4(smem_u32(sQ) + sw_off(r, c), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
        }
    }

    // Base-2 online softmax with an integer base: m_t = running max of the
    // log2-scaled scores, m_r = floor(m_t).  Every rescale is 2^(integer), so
    // bf16(2^(t - m_r)) rescaled later equals bf16(2^(t - final base)) exactly.
    float m_t[2] = {-INFINITY, -INFINITY}, m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
    float o[NDT][4];
#pragma unroll
    for (int i = 0; i < NDT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    for (int it = 0; it < ntiles; ++it) {
        const int st = it % kAttnStages;
        const bool ok = mbar_wait(&bars[st], (uint32_t)((it / kAttnStages) & 1), (volatile int*)&s_abort, p.status);
        if (__syncthreads_or(!ok)) break;   // leave together so the block barriers stay matched
        const int valid = kv1 - (kv0 + it * 64);
        if (valid < 64) {
            // Rows past the last key may hold any bits (never-written cache
            // slack); P is 0 there, but 0 * NaN would poison O, so zero them.
            uint8_t* vs = sV + st * TILE_BYTES;
            for (int idx = tid; idx < (64 - valid) * (D / 8); idx += 128) {
                const int r = valid + idx / (D / 8), c = (idx % (D / 8)) * 8;
                *reinterpret_cast<uint4*>(vs + sw_off(r, c)) = make_uint4(0, 0, 0, 0);
            }
            __syncthreads();
        }
        const uint32_t kb = smem_u32(sK + st * TILE_BYTES), vb = smem_u32(sV + st * TILE_BYTES);
        const int kvbase = kv0 + it * 64 + ks * W;
        // ---- S = Q K^T over this warp's W keys (up to 8 n-tiles of 8 keys)
        float sc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            if (nt * 8 < W) {
                const int r = ks * W + nt * 8 + (lane & 7);
#pragma unroll
                for (int kp = 0; kp < D / 32; ++kp) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4(kb + sw_off(r, kp * 32 + (lane >> 3) * 8), b0, b1, b2, b3);
                    mma_bf16_16816(sc[nt], qa[2 * kp], b0, b1);
                    mma_bf16_16816(sc[nt], qa[2 * kp + 1], b2, b3);
                }
            }
        }
        // ---- online softmax (log2 domain), rows lane/4 and lane/4 + 8
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            if (nt * 8 < W) {
                const int kv = kvbase + nt * 8 + 2 * (lane & 3);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const bool valid_k = (kv + (c & 1)) < kv1;
                    sc[nt][c] = valid_k ? sc[nt][c] * p.scale_log2 : -INFINITY;
                }
                mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
                mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        m_t[0] = fmaxf(m_t[0], mx0);
        m_t[1] = fmaxf(m_t[1], mx1);
        const float nb0 = floorf(m_t[0]), nb1 = floorf(m_t[1]);      // -inf stays -inf
        const float base0 = (nb0 == -INFINITY) ? 0.f : nb0;
        const float base1 = (nb1 == -INFINITY) ? 0.f : nb1;
        const float corr0 = exp2f(m_r[0] - base0), corr1 = exp2f(m_r[1] - base1);   // 0 while m_r is -inf
        m_r[0] = nb0;
        m_r[1] = nb1;
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            if (nt * 8 < W) {
                sc[nt][0] = exp2f(sc[nt][0] - base0);
                sc[nt][1] = exp2f(sc[nt][1] - base0);
                sc[nt][2] = exp2f(sc[nt][2] - base1);
                sc[nt][3] = exp2f(sc[nt][3] - base1);
                ls0 += sc[nt][0] + sc[nt][1];
                ls1 += sc[nt][2] + sc[nt][3];
            }
        }
        l_r[0] = l_r[0] * corr0 + ls0;
        l_r[1] = l_r[1] * corr1 + ls1;
#pragma unroll
        for (int i = 0; i < NDT; ++i) {
            o[i][0] *= corr0;
            o[i][1] *= corr0;
            o[i][2] *= corr1;
            o[i][3] *= corr1;
        }
        // ---- O += P V (P rounded to bf16)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            if (kk * 16 < W) {
                uint32_t pa[4];
                pa[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
                pa[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
                pa[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
                pa[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
                const int r = ks * W + kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
                for (int nd = 0; nd < D / 16; ++nd) {
                    uint32_t b0, b1, b2, b3;
                    ldmatrix_x4_trans(vb + sw_off(r, nd * 16 + (lane >> 4) * 8), b0, b1, b2, b3);
                    mma_bf16_16816(o[2 * nd], pa, b0, b1);
                    mma_bf16_16816(o[2 * nd + 1], pa, b2, b3);
                }
            }
        }
        __syncthreads();
        if (tid == 0 && it + kAttnStages < ntiles && !s_abort) {
            const int nx = it + kAttnStages;
            fence_proxy_async();   // order this stage's generic-proxy accesses before the TMA refill
            mbar_arrive_expect_tx(&bars[st], 2 * TILE_BYTES);
            for (int h = 0; h < D / 64; ++h) {
                tma_load_2d(sK + st * TILE_BYTES + h * 8192, &p.tmap, &bars[st], h * 64, (int)(rowK + kv0 + nx * 64));
                tma_load_2d(sV + st * TILE_BYTES + h * 8192, &p.tmap, &bars[st], h * 64, (int)(rowV + kv0 + nx * 64));
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 1);
        l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 2);
    }
    __syncthreads();   // the ring is free from here on

    // ---- this CTA's partial: merge the key shares of the warps of each row tile
    {
        const int r0 = lane >> 2, c0 = 2 * (lane & 3);
#pragma unroll
        for (int nd = 0; nd < NDT; ++nd) {
            *reinterpret_cast<float2*>(&mo[(warp * 16 + r0) * D + nd * 8 + c0]) = make_float2(o[nd][0], o[nd][1]);
            *reinterpret_cast<float2*>(&mo[(warp * 16 + r0 + 8) * D + nd * 8 + c0]) = make_float2(o[nd][2], o[nd][3]);
        }
        if ((lane & 3) == 0) {
            mml[warp * 16 + r0] = make_float2(m_r[0], l_r[0]);
            mml[warp * 16 + r0 + 8] = make_float2(m_r[1], l_r[1]);
        }
    }
    __syncthreads();
    for (int r = tid; r < R; r += 128) {
        const int t = r >> 4, rr = r & 15;
        float M = -INFINITY;
        for (int k2 = 0; k2 < NKS; ++k2) M = fmaxf(M, mml[(t + k2 * RT) * 16 + rr].x);
        const float base = (M == -INFINITY) ? 0.f : M;
        float L = 0.f;
        for (int k2 = 0; k2 < NKS; ++k2) {
            const float2 ml = mml[(t + k2 * RT) * 16 + rr];
            const float wk = exp2f(ml.x - base);
            wts[r * 4 + k2] = wk;
            L += wk * ml.y;
        }
        pml[r] = make_float2(M, L);
    }
    __syncthreads();
    for (int idx = tid; idx < R * D; idx += 128) {
        const int r = idx / D, c = idx % D, t = r >> 4, rr = r & 15;
        float acc = 0.f;
        for (int k2 = 0; k2 < NKS; ++k2) acc += wts[r * 4 + k2] * mo[((t + k2 * RT) * 16 + rr) * D + c];
        po[r * D + c] = acc;
    }

    // ---- merge the cluster's partials through distributed shared memory
    cluster.sync();
    const float* rpo[kAttnMaxSplits];
    const float2* rpml[kAttnMaxSplits];
#pragma unroll
    for (int s2 = 0; s2 < kAttnMaxSplits; ++s2) {
        rpo[s2] = s2 < nsplit ? cluster.map_shared_rank(po, s2) : po;
        rpml[s2] = s2 < nsplit ? cluster.map_shared_rank(pml, s2) : pml;
    }
    const int nr = r_hi - r_lo;
    for (int idx = tid; idx < nr * nsplit; idx += 128) {
        const int r = r_lo + idx / nsplit, s2 = idx % nsplit;
        const float2 ml = rpml[s2][r];
        cm[idx] = ml.x;
        cl[idx] = ml.y;
    }
    __syncthreads();
    for (int rr = tid; rr < nr; rr += 128) {
        float M = -INFINITY;
        for (int s2 = 0; s2 < nsplit; ++s2) M = fmaxf(M, cm[rr * nsplit + s2]);
        const float base = (M == -INFINITY) ? 0.f : M;
        float L = 0.f;
        for (int s2 = 0; s2 < nsplit; ++s2) {
            const float l = cl[rr * nsplit + s2];
            const float wv = l > 0.f ? exp2f(cm[rr * nsplit + s2] - base) : 0.f;
            cw[rr * nsplit + s2] = wv;
            L += wv * l;
        }
        const float inv = L > 0.f ? 1.0f / L : 0.f;
        for (int s2 = 0; s2 < nsplit; ++s2) cw[rr * nsplit + s2] *= inv;
    }
    __syncthreads();
    for (int idx = tid; idx < nr * D; idx += 128) {
        const int rr = idx / D, c = idx % D, r = r_lo + rr;
        float v[kAttnMaxSplits];
#pragma unroll
        for (int s2 = 0; s2 < kAttnMaxSplits; ++s2) v[s2] = s2 < nsplit ? rpo[s2][r * D + c] : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < kAttnMaxSplits; ++s2)
            if (s2 < nsplit) acc += cw[rr * nsplit + s2] * v[s2];
        const int j = r / p.G, hh = r % p.G;
        p.out[((size_t)(b * p.gamma + j) * p.nq + (size_t)(g * p.G + hh)) * D + c] = f2bf(acc);
    }
    cluster.sync();   // keep this CTA's shared memory alive until every peer has read it
}

int attn_smem_bytes(int d) {
    return 1024 + (1 + 2 * kAttnStages) * 64 * d * 2 + 64;
}

void attn_plan(int B, int nkv, int cap, int num_sms, int& splits, int& chunk) {
    const int tiles = (cap + 63) / 64;
    int s = (num_sms + B * nkv - 1) / (B * nkv);
    s = s < 1 ? 1 : (s > kAttnMaxSplits ? kAttnMaxSplits : s);
    if (s > tiles) s = tiles;
    chunk = ((tiles + s - 1) / s) * 64;
    splits = (cap + chunk - 1) / chunk;
}

int launch_attention(const AttnParams& p, int d, int B, cudaStream_t stream, long long* launches) {
    const int smem = attn_smem_bytes(d);
    void (*kern)(AttnParams) = (d == 128) ? k_attn_cluster<128> : k_attn_cluster<64>;
    static bool done128 = false, done64 = false;
    bool& done = (d == 128) ? done128 : done64;
    if (!done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return (int)e;
        ensure_carveout((const void*)kern);
        done = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.splits, p.nkv, B);
    cfg.blockDim = dim3(128);
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
