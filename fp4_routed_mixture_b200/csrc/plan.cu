// Per-expert work split between the two grouped GEMMs.
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) runs its decode expert GEMMs on
// dot-product instructions and retunes prefill onto matrix cores.  Here the
// choice is made per expert from the sorted offsets: experts with many rows go
// to the tensor-core GEMM (tc_gemm.cu), the others to the streaming GEMM
// (gemv.cu), and this planner writes the scans both launches index.
#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

// Work split per expert: experts with at least tc_min rows go to the
// tensor-core GEMM (tiles of kTcWeightTile weight rows x kTcTokenTile token rows), the others to
// the streaming GEMM (units of 32 weight rows x kGemvGroup tokens).  Writes the
// exclusive scans over experts of the streaming units of W1/W2, of the
// tensor-core tiles of W1/W2 and of the digit-plane rows (each tensor-core
// expert's rows padded to a multiple of 16, so that every tile starts on a
// 16-row boundary of the plane buffers), and expert_tc[e] = 1 for
// tensor-core experts.  One warp; lane l owns a contiguous slice of experts.
__global__ void k_plan(const int32_t* __restrict__ offsets, int E, int P, int n1, int n2, int tc_min,
                       int32_t* __restrict__ unit_off1, int32_t* __restrict__ unit_off2,
                       int32_t* __restrict__ tile_off1, int32_t* __restrict__ tile_off2,
                       int32_t* __restrict__ plane_off, int32_t* __restrict__ expert_tc, int32_t* flag) {
    pdl_begin();
    constexpr int NS = 5;
    const int lane = threadIdx.x;
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    // offsets must run from 0 up to at most P without decreasing; otherwise no
    // expert gets any work (and FLAG_BOUNDS is raised)
    bool bad = (lane == 0 && offsets[0] != 0) || (lane == 31 && offsets[E] > P);
    for (int e = e0; e < e1; ++e) bad |= offsets[e + 1] < offsets[e];
    const bool any_bad = __any_sync(0xffffffffu, bad);
    if (any_bad && lane == 0) raise_flag(flag, FLAG_BOUNDS);
    auto counts = [&](int e, int (&c)[NS]) {
        const int m = any_bad ? 0 : offsets[e + 1] - offsets[e];
        const bool tc = m >= tc_min;
        const int g = tc ? 0 : (m + kGemvGroup - 1) / kGemvGroup;
        const int nb = tc ? (m + kTcTokenTile - 1) / kTcTokenTile : 0;
        c[0] = g * (n1 / 32);
        c[1] = g * (n2 / 32);
        c[2] = nb * (n1 / kTcWeightTile);
        c[3] = nb * (n2 / kTcWeightTile);
        c[4] = tc ? (m + 15) & ~15 : 0;
    };
    int s[NS] = {};
    for (int e = e0; e < e1; ++e) {
        int c[NS];
        counts(e, c);
        for (int j = 0; j < NS; ++j) s[j] += c[j];
    }
    int x[NS];
    for (int j = 0; j < NS; ++j) x[j] = s[j];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int j = 0; j < NS; ++j) {
            const int y = __shfl_up_sync(0xffffffffu, x[j], o);
            if (lane >= o) x[j] += y;
        }
    }
    int r[NS];
    for (int j = 0; j < NS; ++j) r[j] = x[j] - s[j];  // exclusive prefix
    int32_t* outs[NS] = {unit_off1, unit_off2, tile_off1, tile_off2, plane_off};
    for (int e = e0; e < e1; ++e) {
        int c[NS];
        counts(e, c);
        for (int j = 0; j < NS; ++j) {
            outs[j][e] = r[j];
            r[j] += c[j];
        }
        expert_tc[e] = (!any_bad && (offsets[e + 1] - offsets[e]) >= tc_min) ? 1 : 0;
    }
    if (lane == 31)
        for (int j = 0; j < NS; ++j) outs[j][E] = x[j];
}

cudaError_t launch_plan(const int32_t* offsets, int E, int P, int n1, int n2, int tc_min,
                        int32_t* unit_off1, int32_t* unit_off2, int32_t* tile_off1, int32_t* tile_off2,
                        int32_t* plane_off, int32_t* expert_tc, int32_t* flag, cudaStream_t st) {
    const cudaError_t e = launch_pdl(k_plan, dim3(1), dim3(32), 0, st, offsets, E, P, n1, n2, tc_min, unit_off1,
                                     unit_off2, tile_off1, tile_off2, plane_off, expert_tc, flag);
    count_launches(1);
    return e;
}

}  // namespace moe
