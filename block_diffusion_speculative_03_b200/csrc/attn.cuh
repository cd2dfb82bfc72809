// Block attention of the draft step (bf16): parameters and launcher (attn.cu).
#pragma once
#include "common.cuh"

namespace df {

struct AttnParams {
    CUtensorMap tmap;            // cache slab as 2-D [rows, d] bf16, box {64, 64}, 128-byte swizzle
    const __nv_bfloat16* q;      // [B*gamma, nq*d], 16-byte aligned
    __nv_bfloat16* out;          // [B*gamma, nq*d]
    const int* len;
    const int* req_ok;
    int gamma, G, nq, nkv, layer, splits, chunk;
    int causal;                  // 0: every row sees all len + gamma keys; 1: row j sees keys [0, len + j]
    long long rows_req, rows_layer, rows_kind, rows_kv;
    float scale_log2;            // log2(e) / sqrt(d)
    int* status;
    // Diagnostic trace (null in normal use): per CTA 8 globaltimer stamps (ns):
    // entry, past the dependency wait, Q in tensor memory, first tile landed, key loop done,
    // partial ready, past the first cluster barrier, merge done.
    long long* trace;
};

constexpr int kAttnStages = 7;   // K/V ring depth: each stage is held until its tile's P.V is done
constexpr int kAttnThreads = 192;   // TMA warp, MMA warp, 4 softmax warps
constexpr int kAttnMaxSplits = 8;   // CTAs per cluster (portable cluster size)

int attn_smem_bytes(int d);
// Largest cluster the device schedules for the attention kernel (<= kAttnMaxSplits).
int attn_max_cluster(int d);
// Splits (= cluster size) and key rows per split for B requests of `cap` positions.
void attn_plan(int B, int nkv, int cap, int num_sms, int max_cluster, int& splits, int& chunk);
// Launch the cluster kernel: grid (splits, nkv, B), cluster (splits, 1, 1).
int launch_attention(const AttnParams& p, int d, int B, cudaStream_t stream, long long* launches);

}  // namespace df
