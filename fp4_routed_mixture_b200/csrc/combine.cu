// Gate-weighted combine back to token order (the "mixture" of the routed
// mixture-of-experts, "DeepSeek-V4-Flash on AMD gfx90a", abstract):
//   Y[i, n] = fp32(fp64(sh[i]) * acc[i, n])   (streaming-GEMM rows: fp64 sums)
//   Y[i, n] read as is                         (tensor-core rows: final fp32)
//   y[t, n] = bf16( sum_{j<k} gates[t,j] * Y[pos[t*k+j], n] ), fp32, slot order.
// Deterministic gather: each output element is owned by one thread, no atomics.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

__global__ void __launch_bounds__(256)
    k_combine(const double* __restrict__ yacc, const float* __restrict__ yf,
              const int32_t* __restrict__ expert_tc, const int32_t* __restrict__ topk_idx,
              const float* __restrict__ sh, const float* __restrict__ gates,
              const int32_t* __restrict__ pos, int P, int k, int E, int H, __nv_bfloat162* __restrict__ y,
              int32_t* flag) {
    const int t = blockIdx.y;
    const int n2 = blockIdx.x * blockDim.x + threadIdx.x;  // pair of columns
    if (2 * n2 >= H) return;
    float acc0 = 0.0f, acc1 = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int p = t * k + j;
        const int i = checked_index(__ldg(pos + p), P, flag);
        const float g = __ldg(gates + p);
        float y0, y1;
        if (__ldg(expert_tc + checked_index(__ldg(topk_idx + p), E, flag))) {
            const float2 v = __ldg(reinterpret_cast<const float2*>(yf + (size_t)i * H) + n2);
            y0 = v.x;
            y1 = v.y;
        } else {
            const double s = (double)__ldg(sh + i);
            const double2 v = __ldg(reinterpret_cast<const double2*>(yacc + (size_t)i * H) + n2);
            y0 = (float)__dmul_rn(s, v.x);
            y1 = (float)__dmul_rn(s, v.y);
        }
        acc0 = __fmaf_rn(g, y0, acc0);
        acc1 = __fmaf_rn(g, y1, acc1);
    }
    y[(size_t)t * (H / 2) + n2] = __floats2bfloat162_rn(acc0, acc1);
}

cudaError_t launch_combine(const double* yacc, const float* yf, const int32_t* expert_tc,
                           const int32_t* topk_idx, const float* sh, const float* gates,
                           const int32_t* pos, int T, int k, int E, int H, void* y, int32_t* flag,
                           cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    dim3 grid((H / 2 + 255) / 256, T);
    k_combine<<<grid, 256, 0, st>>>(yacc, yf, expert_tc, topk_idx, sh, gates, pos, T * k, k, E, H,
                                    (__nv_bfloat162*)y, flag);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
