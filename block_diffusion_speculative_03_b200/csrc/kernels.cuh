// Launch wrappers of the SIMT kernels (kernels.cu) and the attention kernels (attn.cu).
#pragma once
#include "common.cuh"

namespace df {

struct XSegs {            // X = concat_s seg[s] along k; seg s is [rows, width] with row stride `stride`
    const float* ptr[8];
    long long stride;
    int width;
};

template <typename T>
void launch_embed(const T* embed, const int* anchor, int mask_id, int B, int gamma, int H, int V, const int* len,
                  const int* committed, int cap, T* x, int* req_ok, int* status, cudaStream_t st,
                  long long* tr = nullptr, float* ssq = nullptr);
template <typename T>
void launch_rmsnorm(const T* x, const T* g, T* y, int rows, int H, float eps, int grp, int gstride, int goff,
                    cudaStream_t st, long long* tr = nullptr);
void launch_lm_reduce(const float4* rec, int n_vt, int M, int gm1, const int* req_ok, int* drafts, float* margin,
                      cudaStream_t st, long long* tr = nullptr, int rec_blocks = 0);
void launch_top2_rows(const float* logits, int M, int V, int gm1, const int* req_ok, int* drafts, float* margin,
                      cudaStream_t st);
void launch_accept(const int* drafts, const int* target, int B, int gamma, int V, int* len, int* committed,
                   int* accept_len, int* next_anchor, int* status, cudaStream_t st, long long* tr = nullptr);
void launch_ingest_begin(const __nv_bfloat16* ctx, int B, int rows, int H, const int* len, int cap, __nv_bfloat16* x,
                         int* req_ok, int* status, float* ssq, cudaStream_t st);
void launch_ingest_end(const int* row_count, int rows, int B, const int* req_ok, int* len, int* status,
                       cudaStream_t st);
void launch_inject_finalize(const int* row_count, int B, int cap, int* len, int* status, cudaStream_t st,
                            long long* tr = nullptr);
void launch_set_len(const int* lens, int B, int cap, int* len, int* committed, int* status, cudaStream_t st,
                    long long* tr = nullptr);
int launch_wait_selftest(int* status, int* out, cudaStream_t st);
void launch_synth_target(const int* drafts, const int* a_plan, const int* rnd, int B, int gamma, int V, int* target,
                         cudaStream_t st);
void launch_gemm_f32(const XSegs& xs, const float* W, float* Y, int M, int N, int K, int ldy, int ycol0,
                     cudaStream_t st);
void launch_epi_qkv_f32(const float* Y, int M, int Nq, int Nkv, int d, int gamma, const int* len, const int* req_ok,
                        const float2* rope, float* q, float* slab, long long s_req, long long s_layer, long long s_kind,
                        long long s_kv, int layer, cudaStream_t st);
void launch_epi_inject_f32(const float* Y, int rows, int Nkv, int d, const int* row_start, const int* row_count, int B,
                           const int* len, int cap, const float2* rope, float* slab, long long s_req, long long s_layer,
                           long long s_kind, long long s_kv, int layer, cudaStream_t st);
void launch_resid_f32(float* x, const float* Y, long long n, cudaStream_t st);
void launch_swiglu_f32(const float* Y, float* act, int M, int I, cudaStream_t st);
int launch_attn_f32(const float* q, const float* slab, const int* len, const int* req_ok, float* o, int B, int gamma,
                    int nq, int G, int d, long long s_req, long long s_layer, long long s_kind, long long s_kv,
                    int layer, int cap, cudaStream_t st);

}  // namespace df
