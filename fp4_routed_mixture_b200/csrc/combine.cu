// Gate-weighted combine back to token order (the "mixture" of the routed
// mixture-of-experts, "DeepSeek-V4-Flash on AMD gfx90a", abstract):
//   Y[i, n] = fp32(fp64(sh[i]) * acc[s, n])   (streaming-GEMM rows: fp64 sums
//                                               at the row's streaming row s)
//   Y[i, n] read as is                         (tensor-core rows: final fp32)
//   y[t, n] = bf16( sum_{j<k} gates[t,j] * Y[pos[t*k+j], n] ), fp32, slot order.
// Deterministic gather: each output element is owned by one thread, no atomics.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

// One thread per 4 consecutive columns of one token (16-byte loads of Y).  The
// k slots' row indices, gates and kernel choices are read first and all k rows
// are then loaded before the sum, so the loads overlap.  The kernel choice and
// the compact streaming row come from per-expert tables (expert_tc, offsets,
// stream_off: E entries, cache-resident), not from the per-row slot table, so
// a slot costs no extra dependent miss.  With expert_tc == NULL every row is a
// streaming row stored at its sorted row.  These tables come from the route,
// sort and plan, launches before the h quant (which always runs between them
// and the W2 GEMMs in front of this launch), so they are read before waiting
// on the W2 GEMMs; Y, the fp64 sums and the h scales are read after.
template <int KMAX>
__global__ void __launch_bounds__(256)
    k_combine(const double* __restrict__ yacc, const float* __restrict__ yf,
              const int32_t* __restrict__ expert_tc, const int32_t* __restrict__ offsets,
              const int32_t* __restrict__ stream_off, const int32_t* __restrict__ topk_idx, int E,
              int stream_rows, const float* __restrict__ sh, const float* __restrict__ gates,
              const int32_t* __restrict__ pos, int P, int k, int H, uint2* __restrict__ y, int32_t* flag) {
    const int t = blockIdx.y;
    const int n4 = blockIdx.x * blockDim.x + threadIdx.x;  // group of 4 columns
    if (4 * n4 >= H) return;
    int row[KMAX], srow[KMAX];
    float g[KMAX];
    bool tc[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
            const int p = t * k + j;
            row[j] = checked_index(__ldg(pos + p), P, flag);
            g[j] = __ldg(gates + p);
            tc[j] = false;
            srow[j] = row[j];
            if (expert_tc) {
                const int e = checked_index(__ldg(topk_idx + p), E, flag);
                tc[j] = __ldg(expert_tc + e) != 0;
                if (!tc[j])
                    srow[j] = checked_index(__ldg(stream_off + e) + (row[j] - __ldg(offsets + e)), stream_rows, flag);
            }
        }
    }
    pdl_begin();
    float4 v[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
            if (tc[j]) {
                v[j] = __ldg(reinterpret_cast<const float4*>(yf + (size_t)row[j] * H) + n4);
            } else {
                const double s = (double)__ldg(sh + row[j]);
                const double2* r = reinterpret_cast<const double2*>(yacc + (size_t)srow[j] * H) + 2 * n4;
                const double2 d0 = __ldg(r), d1 = __ldg(r + 1);
                v[j] = make_float4((float)__dmul_rn(s, d0.x), (float)__dmul_rn(s, d0.y), (float)__dmul_rn(s, d1.x),
                                   (float)__dmul_rn(s, d1.y));
            }
        }
    }
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < k) {  // slot order
            acc[0] = __fmaf_rn(g[j], v[j].x, acc[0]);
            acc[1] = __fmaf_rn(g[j], v[j].y, acc[1]);
            acc[2] = __fmaf_rn(g[j], v[j].z, acc[2]);
            acc[3] = __fmaf_rn(g[j], v[j].w, acc[3]);
        }
    }
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
    y[(size_t)t * (H / 4) + n4] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                             *reinterpret_cast<const uint32_t*>(&hi));
}

cudaError_t launch_combine(const double* yacc, const float* yf, const int32_t* expert_tc, const int32_t* offsets,
                           const int32_t* stream_off, const int32_t* topk_idx, int E, int stream_rows,
                           const float* sh, const float* gates, const int32_t* pos, int T, int k, int H, void* y,
                           int32_t* flag, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    dim3 grid((H / 4 + 255) / 256, T);
    const cudaError_t e =
        k <= 8 ? launch_pdl(k_combine<8>, grid, dim3(256), 0, st, yacc, yf, expert_tc, offsets, stream_off,
                            topk_idx, E, stream_rows, sh, gates, pos, T * k, k, H, (uint2*)y, flag)
               : launch_pdl(k_combine<16>, grid, dim3(256), 0, st, yacc, yf, expert_tc, offsets, stream_off,
                            topk_idx, E, stream_rows, sh, gates, pos, T * k, k, H, (uint2*)y, flag);
    count_launches(1);
    return e;
}

}  // namespace moe
