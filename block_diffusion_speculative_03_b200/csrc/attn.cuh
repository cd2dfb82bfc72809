// Block attention of the draft step (bf16): parameters and launcher (attn.cu).
#pragma once
#include "common.cuh"

namespace df {

struct AttnParams {
    CUtensorMap tmap;            // cache slab as 2-D [rows, d] bf16, box {64, 64}, 128-byte swizzle
    const __nv_bfloat16* q;      // [B*gamma, nq*d]
    const int* len;
    const int* req_ok;
    float* part_o;               // [B][nkv][splits][64][d]
    float2* part_ml;             // [B][nkv][splits][64] (row max in log2 units, row sum)
    int gamma, G, nq, nkv, layer, splits, chunk;
    long long rows_req, rows_layer, rows_kind, rows_kv;
    float scale_log2;            // log2(e) / sqrt(d)
    int* status;
};

constexpr int kAttnStages = 2;
// Split count target: two CTAs per SM on a 148-SM B200.
constexpr int kAttnTargetCtas = 296;

int attn_smem_bytes(int d);
// Launch the split kernel and the combine kernel; out = o buffer [B*gamma, nq*d].
int launch_attention(const AttnParams& p, int d, int B, cudaStream_t stream, __nv_bfloat16* out, long long* launches);

}  // namespace df
