// Per-expert work split between the two grouped GEMMs.
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) runs its decode expert GEMMs on
// dot-product instructions and retunes prefill onto matrix cores.  Here the
// choice is made per expert from the sorted offsets: experts with many rows go
// to the tensor-core GEMM (tc_gemm.cu), the others to the streaming GEMM
// (gemv.cu), and this planner (plan_warp in steps.cuh) writes the scans both
// launches index.
#include "steps.cuh"

namespace moe {

// The planner and the per-row state of one layer call, in one launch:
//   every CTA: the plan (warp 0) into shared memory; block 0 publishes it;
//   a thread per sorted row: its slot (kNoRow and steps.cuh): the plane row
//   plane_off[e] + rank inside the expert for rows of tensor-core experts, the
//   complement of its compact streaming row stream_off[e] + rank otherwise; a
//   row whose expert's offsets do not contain it (tables that did not come
//   from one sort) raises FLAG_BOUNDS and gets kNoRow;
//   a CTA per row of a streaming expert: clears its fp64 accumulators (the
//   streaming GEMM adds partial sums into them); skipped when there are none.
// Rows of tensor-core experts are written whole by that GEMM.
__global__ void __launch_bounds__(256)
    k_plan_rows(const int32_t* __restrict__ offsets, const int32_t* __restrict__ topk_idx,
                const int32_t* __restrict__ perm, int E, int P, int I, int H, int tc_min, int tc_tile1, int tc_tile2,
                int tc_wtile1, int tc_wtile2, int group,
                int32_t* __restrict__ unit_off1, int32_t* __restrict__ unit_off2,
                int32_t* __restrict__ tile_off1, int32_t* __restrict__ tile_off2,
                int32_t* __restrict__ plane_off, int32_t* __restrict__ stream_off,
                int32_t* __restrict__ expert_tc, int32_t* __restrict__ plane_row, double* __restrict__ gacc,
                double* __restrict__ yacc, int32_t* flag) {
    pdl_begin();
    __shared__ PlanShared ps;
    if (threadIdx.x < 32)
        plan_warp(offsets, E, P, 2 * I, H, tc_min, tc_tile1, tc_tile2, tc_wtile1, tc_wtile2, group, unit_off1,
                  unit_off2, tile_off1, tile_off2, plane_off, stream_off, expert_tc, flag, blockIdx.x == 0, ps);
    __syncthreads();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < P; i += gridDim.x * blockDim.x) {
        const int e = checked_index(topk_idx[checked_index(perm[i], P, flag)], E, flag);
        const int r0 = offsets[e], r1 = offsets[e + 1];
        int pr = kNoRow;
        if (i >= r0 && i < r1)
            pr = ps.tc[e] ? ps.plane_off[e] + (i - r0) : ~(ps.stream_off[e] + (i - r0));
        else
            raise_flag(flag, FLAG_BOUNDS);
        plane_row[i] = pr;
    }
    if (ps.units1 == 0) return;
    for (int i = blockIdx.x; i < P; i += gridDim.x) {
        const int e = checked_index(topk_idx[checked_index(perm[i], P, flag)], E, flag);
        const int r0 = offsets[e], r1 = offsets[e + 1];
        if (ps.tc[e] || i < r0 || i >= r1) continue;
        const size_t srow = (size_t)(ps.stream_off[e] + (i - r0));
        double2* g = reinterpret_cast<double2*>(gacc + srow * 2 * I);
        for (int j = threadIdx.x; j < I; j += blockDim.x) g[j] = make_double2(0.0, 0.0);
        double2* y = reinterpret_cast<double2*>(yacc + srow * H);
        for (int j = threadIdx.x; j < H / 2; j += blockDim.x) y[j] = make_double2(0.0, 0.0);
    }
}

cudaError_t launch_plan_rows(const int32_t* offsets, const int32_t* topk_idx, const int32_t* perm, int E, int P,
                             int I, int H, int tc_min, int tc_tile1, int tc_tile2, int tc_wtile1, int tc_wtile2,
                             int group, int32_t* unit_off1, int32_t* unit_off2, int32_t* tile_off1,
                             int32_t* tile_off2, int32_t* plane_off, int32_t* stream_off, int32_t* expert_tc,
                             int32_t* plane_row, double* gacc, double* yacc, int32_t* flag, cudaStream_t st) {
    const int grid = std::max(1, std::min(P, 148 * 8));
    const cudaError_t e = launch_pdl(k_plan_rows, dim3(grid), dim3(256), 0, st, offsets, topk_idx, perm, E, P, I,
                                     H, tc_min, tc_tile1, tc_tile2, tc_wtile1, tc_wtile2, group, unit_off1, unit_off2,
                                     tile_off1, tile_off2, plane_off, stream_off, expert_tc, plane_row, gacc, yacc,
                                     flag);
    count_launches(1);
    return e;
}

}  // namespace moe
