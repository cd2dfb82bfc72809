// The split-K tensor-core GEMM with its scratch in a static device array, for
// callers that must not allocate device memory.
//
// dflash_diag_gemm_bf16 takes its split-tile partials and tile counters from
// a buffer the caller allocates.  Some callers cannot provide one: a host that
// owns all device memory through its own pool and hands a library no
// allocator, a serving loop that forbids allocator calls between requests
// (an allocation can synchronise the device or fragment the pool), or code
// that must not grow its footprint after start-up.  For them this variant
// keeps the scratch in a fixed array of this file's module, reserved when the
// library's module loads, and never calls cudaMalloc, cudaFree or any library
// that allocates.
//
// The kernel is the same persistent split-K kernel (gemm_tc.cu); only where
// its scratch lives differs.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/dflash.h"
#include "../../include/dflash_diag.h"
#include "common.cuh"
#include "gemm.cuh"

using namespace df;

namespace {

// Layout of the array: a status word (the kernel's bounded waits record
// DFLASH_TIMEOUT there), padded to 256 bytes; the tile counters (one int per
// output tile, 256-byte aligned); the split-tile partials ([2 * ctas][nt][128]
// fp32).  One array per device: a __device__ variable is instantiated in every
// context that loads the module.
static __device__ __align__(256) unsigned char g_gemm_scratch[DFLASH_NOALLOC_SCRATCH_BYTES];
constexpr size_t kStatusBytes = 256;

constexpr int kMaxDevices = 64;
constexpr int kMaxCtas = 160;
std::mutex g_mu;
struct ScratchAddr {
    CUcontext ctx;   // the context the address was looked up in
    void* ptr;
};
ScratchAddr g_scratch[kMaxDevices] = {};

typedef CUresult (*PFN_ctxGetCurrent_t)(CUcontext*);

// The calling thread's current context (the primary context of the current
// device for runtime-API callers), or nullptr when it cannot be queried.
CUcontext current_context() {
    static PFN_ctxGetCurrent_t fn = nullptr;
    static bool looked = false;
    if (!looked) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_ctxGetCurrent_t)f;
        looked = true;
    }
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

// Device address of this device's array, looked up with that device current
// (the first lookup may load the module into the context).  The address is
// kept per device together with the context it belongs to and looked up again
// whenever the current context is a different one (after a device reset, or
// when the primary context was released and created anew), so a cached address
// never outlives its context.
int scratch_ptr(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return DFLASH_UNSUPPORTED;
    if (cudaFree(nullptr) != cudaSuccess) return DFLASH_CUDA;   // make sure a context is current (allocates nothing)
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lk(g_mu);
    ScratchAddr& a = g_scratch[dev];
    if (!a.ptr || !ctx || a.ctx != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_gemm_scratch) != cudaSuccess || !p) return DFLASH_CUDA;
        a.ptr = p;
        a.ctx = ctx;
    }
    *out = a.ptr;
    return DFLASH_OK;
}

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

}  // namespace

int dflash_diag_gemm_bf16_noalloc(const void* X, const void* W, float* Y, int M, int N, int K, int grid,
                                  dflash_stream stream) {
    if (!X || !W || !Y || M < 1 || M > 4096 || N < 1 || K < 8 || K % 8 || grid < 0) return DFLASH_INVALID_ARG;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DFLASH_CUDA;
    const int nt = pick_nt(M);
    const long long tiles = (long long)ceil_div(N, 128) * ceil_div(M, nt);
    const long long units = tiles * ceil_div(K, 64);
    // the CTA count the launcher will use (it never exceeds the unit count)
    int ctas = std::min(sms, kMaxCtas);
    if (grid > 0) ctas = std::min(grid, ctas);
    if ((long long)ctas > units) ctas = (int)units;
    const size_t counter_bytes = round_up((size_t)tiles * sizeof(int), 256);
    const size_t need = kStatusBytes + counter_bytes + gemm_partial_bytes(ctas, nt);
    if (need > (size_t)DFLASH_NOALLOC_SCRATCH_BYTES) return DFLASH_WORKSPACE;

    void* scratch = nullptr;
    int st = scratch_ptr(dev, &scratch);
    if (st != DFLASH_OK) return st;

    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    if (!encode_bf16_2d(&p.ta[0], W, K, N, K, 128) || !encode_bf16_2d(&p.tb[0], X, K, M, K, nt))
        return DFLASH_INVALID_ARG;
    p.amat[0].rows = N;
    p.n_amat = 1;
    p.kb_per_b = ceil_div(K, 64);
    p.M = M;
    p.K = K;
    p.epi = EPI_F32;
    p.out = Y;
    p.ldo = N;
    p.status = (int*)scratch;
    p.counters = (int*)((unsigned char*)scratch + kStatusBytes);
    p.partial = (float*)((unsigned char*)scratch + kStatusBytes + counter_bytes);
    p.trace = nullptr;
    p.ctas = ctas;   // the scratch above is sized for exactly this many CTAs
    cudaStream_t s = (cudaStream_t)stream;
    // The array keeps whatever the previous call left.  The kernel returns
    // the counters to zero, but a call that stopped early (a timed-out wait)
    // would leave them set, so they are cleared here together with the status
    // word; the partials are always written before they are read and need no
    // clearing.
    if (cudaMemsetAsync(scratch, 0, kStatusBytes + counter_bytes, s) != cudaSuccess) return DFLASH_CUDA;
    return launch_gemm_tc(p, nt, std::min(sms, kMaxCtas), s) == 0 ? DFLASH_OK : DFLASH_CUDA;
}

int dflash_diag_gemm_bf16_noalloc_status(int32_t* status, dflash_stream stream) {
    if (!status) return DFLASH_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DFLASH_CUDA;
    void* scratch = nullptr;
    int st = scratch_ptr(dev, &scratch);
    if (st != DFLASH_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    int word = 0;
    if (cudaMemcpyAsync(&word, scratch, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return DFLASH_CUDA;
    *status = word;
    return DFLASH_OK;
}
