// Expert sorting: stable counting sort of token-expert pairs by expert.
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) groups the routed pairs by
// expert before the expert GEMMs and retunes that sort for prefill.  Here the
// sort is an atomic histogram in shared memory, a prefix scan, and a stable
// scatter:
//   k_sort_count   (one CTA per chunk of 1024 pairs): per-chunk histogram
//   k_sort_scatter (one CTA per chunk): every CTA rebuilds the global offsets
//                  and its chunk's starting cursor per expert from the chunk
//                  histograms, then one warp walks the chunk in pair order;
//                  __match_any_sync ranks equal experts inside each 32-pair
//                  step, which keeps the sort stable.
// A single chunk (P <= 1024, the decode case) runs both phases in one launch.
// Expert ids outside [0, E) raise FLAG_BAD_EXPERT and are skipped.
#include "steps.cuh"

namespace moe {

__global__ void __launch_bounds__(kSortThreads)
    k_sort_count(const int32_t* __restrict__ topk_idx, int P, int E, int32_t* __restrict__ chunk_hist,
                 int32_t* flag) {
    pdl_begin();
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int p0 = blockIdx.x * kSortChunk, p1 = min(P, p0 + kSortChunk);
    bool bad = false;
    for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
        const int e = __ldg(topk_idx + p);
        if (valid_expert(e, E))
            atomicAdd(&hist[e], 1);
        else
            bad = true;
    }
    if (bad) raise_flag(flag, FLAG_BAD_EXPERT);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_hist[(size_t)blockIdx.x * E + e] = hist[e];
}

__global__ void __launch_bounds__(kSortThreads)
    k_sort_scatter(const int32_t* __restrict__ topk_idx, int P, int E,
                   const int32_t* __restrict__ chunk_hist, int32_t* __restrict__ perm,
                   int32_t* __restrict__ pos, int32_t* __restrict__ offsets) {
    pdl_begin();
    extern __shared__ int sm[];
    int* total = sm;           // [E] -> exclusive offsets
    int* cursor = sm + E;      // [E]
    int* tmp = sm + 2 * E;     // [kSortThreads + 1]
    const int nchunks = gridDim.x, c = blockIdx.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int tot = 0, before = 0;
#pragma unroll 8
        for (int j = 0; j < nchunks; ++j) {
            const int v = chunk_hist[(size_t)j * E + e];
            tot += v;
            if (j < c) before += v;
        }
        total[e] = tot;
        cursor[e] = before;
    }
    __syncthreads();
    const int all = block_exclusive_scan(total, E, tmp);
    for (int e = threadIdx.x; e < E; e += blockDim.x) cursor[e] += total[e];
    if (c == 0) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) offsets[e] = total[e];
        if (threadIdx.x == 0) offsets[E] = all;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int p0 = c * kSortChunk, p1 = min(P, p0 + kSortChunk);
        warp_stable_scatter([&](int p) { return (int)__ldg(topk_idx + p); }, p0, p1, E, cursor, perm, pos);
    }
}

// P <= kSortChunk: histogram, scan and scatter in one CTA (sort_cta).
__global__ void __launch_bounds__(kSortThreads)
    k_sort_single(const int32_t* __restrict__ topk_idx, int P, int E, int32_t* __restrict__ perm,
                  int32_t* __restrict__ pos, int32_t* __restrict__ offsets, int32_t* flag) {
    pdl_begin();
    extern __shared__ int sm[];
    if (threadIdx.x == 0) *flag = 0;  // this single CTA is the whole sort: it owns the error word
    sort_cta([&](int p) { return (int)__ldg(topk_idx + p); }, P, E, perm, pos, offsets, sm, sm + E, nullptr,
             flag);
}

size_t sort_workspace_bytes(int T_max, int k, int E) {
    const size_t P = (size_t)T_max * k;
    const size_t chunks = (P + kSortChunk - 1) / kSortChunk;
    return 256 + align_up(std::max<size_t>(chunks, 1) * E * sizeof(int32_t), 256);
}

cudaError_t launch_sort(const int32_t* topk_idx, int T, int k, int E, int32_t* perm, int32_t* pos,
                        int32_t* offsets, void* ws, cudaStream_t st) {
    int32_t* flag = (int32_t*)ws;
    int32_t* chunk_hist = (int32_t*)((char*)ws + 256);
    const int P = T * k;
    if (P <= kSortChunk) {  // k_sort_single clears the error word itself
        const size_t smem = (size_t)(E + kSortThreads + 1) * sizeof(int);
        const cudaError_t e = launch_pdl(k_sort_single, dim3(1), dim3(kSortThreads), smem, st, topk_idx, P, E,
                                         perm, pos, offsets, flag);
        count_launches(1);
        return e;
    }
    cudaError_t err = cudaMemsetAsync(flag, 0, sizeof(int32_t), st);
    if (err != cudaSuccess) return err;
    const int chunks = (P + kSortChunk - 1) / kSortChunk;
    err = launch_pdl(k_sort_count, dim3(chunks), dim3(kSortThreads), (size_t)E * sizeof(int), st, topk_idx, P, E,
                     chunk_hist, flag);
    count_launches(1);
    if (err != cudaSuccess) return err;
    const size_t smem = (size_t)(2 * E + kSortThreads + 1) * sizeof(int);
    err = launch_pdl(k_sort_scatter, dim3(chunks), dim3(kSortThreads), smem, st, topk_idx, P, E,
                     (const int32_t*)chunk_hist, perm, pos, offsets);
    count_launches(1);
    return err;
}

// ---- the same sort with library-owned scratch (moe_sort_static) -------------
// For callers that are handed only input and output pointers and have no way
// to obtain a device workspace: the scratch (error word + per-chunk
// histograms) lives in this file-scope device array.  Every GPU that loads the
// library holds it until the process exits; every call shares it, so calls
// that overlap on a GPU race.  It keeps the previous call's contents: the
// error word is cleared by every call and every histogram entry a call reads
// is written by that same call first.
constexpr int kSortStaticMaxPairs = 65536;
constexpr int kSortStaticMaxExperts = 1024;
constexpr size_t kSortStaticBytes =
    256 + (size_t)(kSortStaticMaxPairs / kSortChunk) * kSortStaticMaxExperts * sizeof(int32_t);
static __device__ __align__(256) uint8_t g_sort_scratch[kSortStaticBytes];

static_assert(kSortStaticMaxPairs % kSortChunk == 0, "whole chunks");
static_assert(kSortChunk <= 32 * 32, "warp_stable_scatter holds 32 ids per lane");

// Device address of g_sort_scratch in the calling thread's current context.
// The host-side name is only a stand-in; the address belongs to this
// library's module as loaded in that context, which a cudaDeviceReset or a
// caller-created context replaces, so it is looked up on every call (a host
// table lookup once the module is loaded).
static cudaError_t sort_static_scratch(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_sort_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

int sort_static_fits(int T, int k, int E) {
    return (long long)T * k <= kSortStaticMaxPairs && E <= kSortStaticMaxExperts;
}

cudaError_t launch_sort_static(const int32_t* topk_idx, int T, int k, int E, int32_t* perm,
                               int32_t* pos, int32_t* offsets, cudaStream_t st) {
    void* ws = nullptr;
    cudaError_t e = sort_static_scratch(&ws);
    if (e != cudaSuccess) return e;
    return launch_sort(topk_idx, T, k, E, perm, pos, offsets, ws, st);
}

}  // namespace moe
