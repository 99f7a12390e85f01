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
// tensor-core GEMM (tiles of kTcWeightTile weight rows x kTcTokenTile token
// rows), the others to the streaming GEMM (units of 32 weight rows x
// kGemvGroup tokens).  Forms the exclusive scans over experts of the streaming
// units of W1/W2, of the tensor-core tiles of W1/W2 and of the digit-plane rows
// (each tensor-core expert's rows padded to a multiple of 16, so that every
// tile starts on a 16-row boundary of the plane buffers), and expert_tc[e] = 1
// for tensor-core experts.  Run by one warp; lane l owns a contiguous slice of
// experts.  Every CTA of k_plan_rows runs it into its shared memory (the row
// pass below needs the tables at once, and the warp's work is small); block 0
// also writes the global tables the GEMM launches index.
struct PlanShared {
    int32_t plane_off[kMaxExperts];
    uint8_t tc[kMaxExperts];
    int32_t units1;   // streaming units of W1 (0: no streaming rows)
};

__device__ void plan_warp(const int32_t* __restrict__ offsets, int E, int P, int n1, int n2, int tc_min,
                          int32_t* __restrict__ unit_off1, int32_t* __restrict__ unit_off2,
                          int32_t* __restrict__ tile_off1, int32_t* __restrict__ tile_off2,
                          int32_t* __restrict__ plane_off, int32_t* __restrict__ expert_tc, int32_t* flag,
                          bool global_out, PlanShared& ps) {
    constexpr int NS = 5;
    const int lane = threadIdx.x & 31;
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    // offsets must run from 0 up to at most P without decreasing; otherwise no
    // expert gets any work (and FLAG_BOUNDS is raised)
    bool bad = (lane == 0 && offsets[0] != 0) || (lane == 31 && offsets[E] > P);
    for (int e = e0; e < e1; ++e) bad |= offsets[e + 1] < offsets[e];
    const bool any_bad = __any_sync(0xffffffffu, bad);
    if (any_bad && lane == 0 && global_out) raise_flag(flag, FLAG_BOUNDS);
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
        const bool tc = !any_bad && (offsets[e + 1] - offsets[e]) >= tc_min;
        ps.plane_off[e] = r[4];
        ps.tc[e] = tc ? 1 : 0;
        if (global_out) {
            for (int j = 0; j < NS; ++j) outs[j][e] = r[j];
            expert_tc[e] = tc ? 1 : 0;
        }
        for (int j = 0; j < NS; ++j) r[j] += c[j];
    }
    if (lane == 31) {
        ps.units1 = x[0];
        if (global_out)
            for (int j = 0; j < NS; ++j) outs[j][E] = x[j];
    }
}

// The planner and the per-row state of one layer call, in one launch:
//   every CTA: the plan (warp 0) into shared memory; block 0 publishes it;
//   a thread per sorted row: its plane row (plane_off[e] + rank inside the
//   expert) for rows of tensor-core experts, -1 otherwise; a row whose expert's
//   offsets do not contain it (tables that did not come from one sort) raises
//   FLAG_BOUNDS and gets no plane row;
//   a CTA per row of a streaming expert: clears its fp64 accumulators (the
//   streaming GEMM adds partial sums into them); skipped when there are none.
// Rows of tensor-core experts are written whole by that GEMM.
__global__ void __launch_bounds__(256)
    k_plan_rows(const int32_t* __restrict__ offsets, const int32_t* __restrict__ topk_idx,
                const int32_t* __restrict__ perm, int E, int P, int I, int H, int tc_min,
                int32_t* __restrict__ unit_off1, int32_t* __restrict__ unit_off2,
                int32_t* __restrict__ tile_off1, int32_t* __restrict__ tile_off2,
                int32_t* __restrict__ plane_off, int32_t* __restrict__ expert_tc,
                int32_t* __restrict__ plane_row, double* __restrict__ gacc, double* __restrict__ yacc,
                int32_t* flag) {
    pdl_begin();
    __shared__ PlanShared ps;
    if (threadIdx.x < 32)
        plan_warp(offsets, E, P, 2 * I, H, tc_min, unit_off1, unit_off2, tile_off1, tile_off2, plane_off,
                  expert_tc, flag, blockIdx.x == 0, ps);
    __syncthreads();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < P; i += gridDim.x * blockDim.x) {
        const int e = checked_index(topk_idx[checked_index(perm[i], P, flag)], E, flag);
        int pr = -1;
        if (ps.tc[e]) {
            const int r0 = offsets[e], r1 = offsets[e + 1];
            if (i >= r0 && i < r1)
                pr = ps.plane_off[e] + (i - r0);
            else
                raise_flag(flag, FLAG_BOUNDS);
        }
        plane_row[i] = pr;
    }
    if (ps.units1 == 0) return;
    for (int i = blockIdx.x; i < P; i += gridDim.x) {
        const int e = checked_index(topk_idx[checked_index(perm[i], P, flag)], E, flag);
        if (ps.tc[e]) continue;
        double2* g = reinterpret_cast<double2*>(gacc + (size_t)i * 2 * I);
        for (int j = threadIdx.x; j < I; j += blockDim.x) g[j] = make_double2(0.0, 0.0);
        double2* y = reinterpret_cast<double2*>(yacc + (size_t)i * H);
        for (int j = threadIdx.x; j < H / 2; j += blockDim.x) y[j] = make_double2(0.0, 0.0);
    }
}

cudaError_t launch_plan_rows(const int32_t* offsets, const int32_t* topk_idx, const int32_t* perm, int E, int P,
                             int I, int H, int tc_min, int32_t* unit_off1, int32_t* unit_off2,
                             int32_t* tile_off1, int32_t* tile_off2, int32_t* plane_off, int32_t* expert_tc,
                             int32_t* plane_row, double* gacc, double* yacc, int32_t* flag, cudaStream_t st) {
    const int grid = std::max(1, std::min(P, 148 * 8));
    const cudaError_t e = launch_pdl(k_plan_rows, dim3(grid), dim3(256), 0, st, offsets, topk_idx, perm, E, P, I,
                                     H, tc_min, unit_off1, unit_off2, tile_off1, tile_off2, plane_off, expert_tc,
                                     plane_row, gacc, yacc, flag);
    count_launches(1);
    return e;
}

}  // namespace moe
