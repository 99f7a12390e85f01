// The steps before the first expert GEMM of a decode-size layer call, fused
// into one launch.
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) names per-layer
// synchronisation among the costs of its decode path.  At decode the route,
// sort, x quant and plan steps each move a few kilobytes, so as separate
// launches their time is mostly launch and dependency latency.  When no expert
// can reach the tensor-core threshold (T below it: every expert has at most T
// rows) and the pairs fit one sort chunk, one launch runs them all, with
// roles by block:
//   block 0      routes every token (a warp per token, route_token), sorts the
//                pairs (sort_cta, expert ids from shared memory) and forms the
//                streaming-unit scans (front_plan_warp); it also owns the
//                call's error word (cleared, FLAG_LAYOUT on a packed-header
//                mismatch);
//   blocks 1..T  x quant of token blockIdx.x - 1 (xquant_row);
//   the rest     clear the fp64 accumulators of one sorted row each (every
//                row is a streaming row here).
// No role reads another's output, so no block waits for another; the first
// GEMM waits for the whole grid (programmatic dependent launch) exactly as it
// waited for the four launches this replaces.  The results are the same as
// those of k_route, k_sort_single, k_xquant and k_plan_rows.
#include "steps.cuh"

namespace moe {

struct FrontArgs {
    const float* logits;        // [T, E]
    const __nv_bfloat16* x;     // [T, H]
    const void* packed;
    int T, H, I, E, k;
    int group;                  // token rows per streaming-GEMM unit
    int32_t* topk_idx;          // [T, k]
    float* gates;               // [T, k]
    int32_t* perm;              // [P]
    int32_t* pos;               // [P]
    int32_t* offsets;           // [E + 1]
    int32_t *unit_off1, *unit_off2, *plane_row;
    int8_t* xq;
    float* sx;
    int32_t* xinit;
    int8_t* dbg_xq;
    float* dbg_sx;
    double* gacc;               // [P, 2I]
    double* yacc;               // [P, H]
    int32_t* flag;
};

// The streaming-unit scans of a call in which every expert takes the
// streaming GEMM: unit_off1[e] / unit_off2[e] = (token groups of the experts
// before e) x (weight tiles of W1 / W2), [E] the totals.  One warp; lane l
// owns a contiguous slice of experts.
__device__ __forceinline__ void front_plan_warp(const int* offs, int E, int group, int tiles1, int tiles2,
                                                int32_t* __restrict__ unit_off1, int32_t* __restrict__ unit_off2) {
    const int lane = threadIdx.x & 31;
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int s = 0;
    for (int e = e0; e < e1; ++e) s += (offs[e + 1] - offs[e] + group - 1) / group;
    int x = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    int run = x - s;
    for (int e = e0; e < e1; ++e) {
        unit_off1[e] = run * tiles1;
        unit_off2[e] = run * tiles2;
        run += (offs[e + 1] - offs[e] + group - 1) / group;
    }
    if (lane == 31) {
        unit_off1[E] = x * tiles1;
        unit_off2[E] = x * tiles2;
    }
}

template <int KMAX, int S>
__global__ void __launch_bounds__(kSortThreads) k_layer_front(FrontArgs a) {
    pdl_begin();
    const int P = a.T * a.k;
    if (blockIdx.x == 0) {
        __shared__ int s_idx[kFrontMaxPairs];
        __shared__ int hist[kMaxExperts];
        __shared__ int tmp[kSortThreads + 1];
        __shared__ int offs[kMaxExperts + 1];
        if (threadIdx.x == 0) *a.flag = packed_header_ok(a.packed, a.H, a.I, a.E) ? 0 : FLAG_LAYOUT;
        const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
        for (int t = warp; t < a.T; t += nwarps)
            route_token<KMAX, S>(a.logits + (size_t)t * a.E, a.E, a.k, a.topk_idx + (size_t)t * a.k,
                                 a.gates + (size_t)t * a.k, s_idx + t * a.k);
        __syncthreads();
        sort_cta([&](int p) { return s_idx[p]; }, P, a.E, a.perm, a.pos, a.offsets, hist, tmp, offs, a.flag);
        __syncthreads();
        // no expert reaches the tensor-core threshold, so the only tables the
        // launches of this call read are the streaming units of W1 and W2
        // (units of an expert: its token groups times the weight tiles) and
        // the streaming rows, which are the sorted offsets themselves
        if (threadIdx.x < 32) front_plan_warp(offs, a.E, a.group, 2 * a.I / kGemvTileRows, a.H / kGemvTileRows,
                                              a.unit_off1, a.unit_off2);
        // every row is a streaming row and every expert's streaming rows start
        // at its sorted offset, so sorted row i is streaming row i
        for (int i = threadIdx.x; i < P; i += blockDim.x) a.plane_row[i] = ~i;
        return;
    }
    if ((int)blockIdx.x <= a.T) {
        __shared__ float red[33];
        __shared__ uint16_t lut[256];
        xquant_row(a.x, (int)blockIdx.x - 1, a.H, a.xq, a.sx, a.xinit, nullptr, a.dbg_xq, a.dbg_sx, red, lut);
        return;
    }
    const int i = (int)blockIdx.x - 1 - a.T;  // sorted row (grid: 1 + T + P blocks)
    double2* g = reinterpret_cast<double2*>(a.gacc + (size_t)i * 2 * a.I);
    for (int j = threadIdx.x; j < a.I; j += blockDim.x) g[j] = make_double2(0.0, 0.0);
    double2* y = reinterpret_cast<double2*>(a.yacc + (size_t)i * a.H);
    for (int j = threadIdx.x; j < a.H / 2; j += blockDim.x) y[j] = make_double2(0.0, 0.0);
}

cudaError_t launch_layer_front(const float* logits, const void* x, const void* packed, int T, int H, int I,
                               int E, int k, int group, int32_t* topk_idx, float* gates, int32_t* perm, int32_t* pos,
                               int32_t* offsets, int32_t* unit_off1, int32_t* unit_off2, int32_t* plane_row, int8_t* xq, float* sx, int32_t* xinit, int8_t* dbg_xq,
                               float* dbg_sx, double* gacc, double* yacc, int32_t* flag, cudaStream_t st) {
    const int P = T * k;
    if (T < 1 || P > kFrontMaxPairs || E > kMaxExperts) return cudaErrorInvalidValue;
    FrontArgs a{logits, (const __nv_bfloat16*)x, packed, T, H, I, E, k, group, topk_idx, gates, perm, pos, offsets,
                unit_off1, unit_off2, plane_row, xq, sx, xinit,
                dbg_xq, dbg_sx, gacc, yacc, flag};
    const dim3 grid(1 + T + P), block(kSortThreads);
    cudaError_t e;
    if (E <= 256)
        e = k <= 8 ? launch_pdl(k_layer_front<8, 8>, grid, block, 0, st, a)
                   : launch_pdl(k_layer_front<16, 8>, grid, block, 0, st, a);
    else
        e = k <= 8 ? launch_pdl(k_layer_front<8, 32>, grid, block, 0, st, a)
                   : launch_pdl(k_layer_front<16, 32>, grid, block, 0, st, a);
    count_launches(1);
    return e;
}

}  // namespace moe
