// Block attention of the draft step (bf16 storage), split over the key axis.
//
// For request b and kv head g, the G*gamma query rows (G = query heads per kv
// head) attend to every cached row [0, len) plus the gamma block rows that the
// QKV epilogue wrote at [len, len+gamma): no mask.  CTA (split s, g, b) takes
// key rows [s*chunk, (s+1)*chunk): K/V tiles of 64 rows x d arrive by TMA
// (128-byte swizzle, no multicast) into a 2-stage ring; each warp owns 16
// query rows (and a share of each tile's keys when there are fewer than 64
// rows), computes S = Q K^T and O += P V with mma.sync m16n8k16 (bf16 in, fp32
// accumulate), and keeps the online-softmax row max / sum with quad shuffles.
// Partials (m, l, O) per split are merged by k_attn_combine.
#include "attn.cuh"

namespace df {




// Byte offset of element (r, c) in a [64 rows][D] bf16 tile stored as D/64
// column blocks of [64 rows][128 B] with the 128-byte swizzle (16-byte chunk
// index XOR row % 8), which is the layout TMA writes.
DF_DEV uint32_t sw_off(int r, int c) {
    return (uint32_t)((c >> 6) * (64 * 128) + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1));
}

template <int D>
__global__ void __launch_bounds__(128) k_attn_split(const __grid_constant__ AttnParams p) {
    constexpr int TILE_BYTES = 64 * D * 2;
    constexpr int NDT = D / 8;     // n-tiles of the output
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sQ = smem;
    uint8_t* sK = sQ + TILE_BYTES;                   // [stages]
    uint8_t* sV = sK + kAttnStages * TILE_BYTES;     // [stages]
    uint64_t* bars = (uint64_t*)(sV + kAttnStages * TILE_BYTES);
    __shared__ int s_abort;

    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (!p.req_ok[b]) return;
    const int n = p.len[b] + p.gamma;
    const int kv0 = s * p.chunk;
    const int kv1 = min(n, kv0 + p.chunk);
    const int ntiles = kv1 > kv0 ? (kv1 - kv0 + 63) / 64 : 0;
    const int R = p.G * p.gamma;
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
        tma_prefetch_desc(&p.tmap);
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

    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
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
                    const bool valid = (kv + (c & 1)) < kv1;
                    sc[nt][c] = valid ? sc[nt][c] * p.scale_log2 : -INFINITY;
                }
                mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
                mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m_r[0], mx0), mn1 = fmaxf(m_r[1], mx1);
        const float base0 = (mn0 == -INFINITY) ? 0.f : mn0;
        const float base1 = (mn1 == -INFINITY) ? 0.f : mn1;
        const float corr0 = exp2f(m_r[0] - base0), corr1 = exp2f(m_r[1] - base1);
        m_r[0] = mn0;
        m_r[1] = mn1;
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
    // Quad-reduce the row sums.
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 1);
        l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 2);
    }
    __syncthreads();
    // Merge the key shares of warps that hold the same query rows.
    float* mo = (float*)(smem + TILE_BYTES);          // reuse the K/V ring: [4 warps][16][D]
    float* mml = mo + 4 * 16 * D;                     // [4 warps][16][2]
    if (NKS > 1) {
        const int r0 = lane >> 2, c0 = 2 * (lane & 3);
#pragma unroll
        for (int nd = 0; nd < NDT; ++nd) {
            mo[(warp * 16 + r0) * D + nd * 8 + c0] = o[nd][0];
            mo[(warp * 16 + r0) * D + nd * 8 + c0 + 1] = o[nd][1];
            mo[(warp * 16 + r0 + 8) * D + nd * 8 + c0] = o[nd][2];
            mo[(warp * 16 + r0 + 8) * D + nd * 8 + c0 + 1] = o[nd][3];
        }
        if ((lane & 3) == 0) {
            mml[(warp * 16 + r0) * 2] = m_r[0];
            mml[(warp * 16 + r0) * 2 + 1] = l_r[0];
            mml[(warp * 16 + r0 + 8) * 2] = m_r[1];
            mml[(warp * 16 + r0 + 8) * 2 + 1] = l_r[1];
        }
        __syncthreads();
        if (ks == 0) {
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int r = (lane >> 2) + hr * 8;
                float M = -INFINITY;
                for (int k2 = 0; k2 < NKS; ++k2) M = fmaxf(M, mml[((rt + k2 * RT) * 16 + r) * 2]);
                const float base = (M == -INFINITY) ? 0.f : M;
                float L = 0.f;
                float sc2[4];
                for (int k2 = 0; k2 < NKS; ++k2) {
                    sc2[k2] = exp2f(mml[((rt + k2 * RT) * 16 + r) * 2] - base);
                    L += sc2[k2] * mml[((rt + k2 * RT) * 16 + r) * 2 + 1];
                }
#pragma unroll
                for (int nd = 0; nd < NDT; ++nd) {
                    for (int cc = 0; cc < 2; ++cc) {
                        float acc = 0.f;
                        for (int k2 = 0; k2 < NKS; ++k2)
                            acc += sc2[k2] * mo[((rt + k2 * RT) * 16 + r) * D + nd * 8 + 2 * (lane & 3) + cc];
                        o[nd][hr * 2 + cc] = acc;
                    }
                }
                m_r[hr] = M;
                l_r[hr] = L;
            }
        }
    }
    if (ks == 0) {
        const size_t base = ((size_t)(b * p.nkv + g) * p.splits + s) * 64;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int r = rt * 16 + (lane >> 2) + hr * 8;
            if (r < R) {
                float* dst = p.part_o + (base + r) * D;
#pragma unroll
                for (int nd = 0; nd < NDT; ++nd)
                    *reinterpret_cast<float2*>(dst + nd * 8 + 2 * (lane & 3)) = make_float2(o[nd][hr * 2], o[nd][hr * 2 + 1]);
                if ((lane & 3) == 0) p.part_ml[base + r] = make_float2(m_r[hr], l_r[hr]);
            }
        }
    }
}

// Merge the split partials: one warp per (request, block position, query head).
template <int D>
__global__ void k_attn_combine(const float* __restrict__ part_o, const float2* __restrict__ part_ml,
                               __nv_bfloat16* __restrict__ out, const int* __restrict__ req_ok, int B, int gamma,
                               int G, int nq, int nkv, int splits) {
    const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (wid >= B * gamma * nq) return;
    const int hq = wid % nq, j = (wid / nq) % gamma, b = wid / (nq * gamma);
    const int g = hq / G, r = j * G + (hq % G);
    constexpr int PER = D / 32;
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
    __nv_bfloat16* dst = out + ((size_t)(b * gamma + j) * nq + hq) * D;
    if (!req_ok[b]) {
        for (int i = 0; i < PER; ++i) dst[lane + 32 * i] = f2bf(0.f);
        return;
    }
    const size_t base = (size_t)(b * nkv + g) * splits * 64 + r;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, part_ml[base + (size_t)s * 64].x);
    const float mb = (M == -INFINITY) ? 0.f : M;
    float L = 0.f;
    for (int s = 0; s < splits; ++s) {
        const float2 ml = part_ml[base + (size_t)s * 64];
        if (ml.y == 0.f) continue;
        const float w = exp2f(ml.x - mb);
        L += w * ml.y;
        const float* po = part_o + (base + (size_t)s * 64) * D;
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] += w * po[lane + 32 * i];
    }
    const float inv = L > 0.f ? 1.0f / L : 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) dst[lane + 32 * i] = f2bf(acc[i] * inv);
}

int attn_smem_bytes(int d) { return 1024 + (1 + 2 * kAttnStages) * 64 * d * 2 + 64; }

int launch_attention(const AttnParams& p, int d, int B, cudaStream_t stream, __nv_bfloat16* out,
                     long long* launches) {
    dim3 grid(p.splits, p.nkv, B);
    const int smem = attn_smem_bytes(d);
    cudaError_t e;
    if (d == 128) {
        static bool done = false;
        if (!done) {
            e = cudaFuncSetAttribute(k_attn_split<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return (int)e;
            done = true;
        }
        k_attn_split<128><<<grid, 128, smem, stream>>>(p);
    } else {
        static bool done = false;
        if (!done) {
            e = cudaFuncSetAttribute(k_attn_split<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return (int)e;
            done = true;
        }
        k_attn_split<64><<<grid, 128, smem, stream>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
    const int warps = B * p.gamma * p.nq;
    const int blocks = (warps * 32 + 255) / 256;
    if (d == 128)
        k_attn_combine<128><<<blocks, 256, 0, stream>>>(p.part_o, p.part_ml, out, p.req_ok, B, p.gamma, p.G, p.nq,
                                                        p.nkv, p.splits);
    else
        k_attn_combine<64><<<blocks, 256, 0, stream>>>(p.part_o, p.part_ml, out, p.req_ok, B, p.gamma, p.G, p.nq,
                                                       p.nkv, p.splits);
    *launches += 2;
    return (int)cudaGetLastError();
}

}  // namespace df
