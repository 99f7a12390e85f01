// Gate-weighted combine back to token order (the "mixture" of the routed
// mixture-of-experts, "DeepSeek-V4-Flash on AMD gfx90a", abstract):
//   Y[i, n] = fp32(fp64(sh[i]) * acc[i, n])          (W2 output of sorted row i)
//   y[t, n] = bf16( sum_{j<k} gates[t,j] * Y[pos[t*k+j], n] ), fp32, slot order.
// Deterministic gather: each output element is owned by one thread, no atomics.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

__global__ void __launch_bounds__(256)
    k_combine(const double* __restrict__ yacc, const float* __restrict__ sh,
              const float* __restrict__ gates, const int32_t* __restrict__ pos, int k, int H,
              __nv_bfloat162* __restrict__ y) {
    const int t = blockIdx.y;
    const int n2 = blockIdx.x * blockDim.x + threadIdx.x;  // pair of columns
    if (2 * n2 >= H) return;
    float acc0 = 0.0f, acc1 = 0.0f;
    for (int j = 0; j < k; ++j) {
        const int i = __ldg(pos + (size_t)t * k + j);
        const float g = __ldg(gates + (size_t)t * k + j);
        const double s = (double)__ldg(sh + i);
        const double2 a = __ldg(reinterpret_cast<const double2*>(yacc + (size_t)i * H) + n2);
        acc0 = __fmaf_rn(g, (float)__dmul_rn(s, a.x), acc0);
        acc1 = __fmaf_rn(g, (float)__dmul_rn(s, a.y), acc1);
    }
    y[(size_t)t * (H / 2) + n2] = __floats2bfloat162_rn(acc0, acc1);
}

cudaError_t launch_combine(const double* yacc, const float* sh, const float* gates,
                           const int32_t* pos, int T, int k, int H, void* y, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    dim3 grid((H / 2 + 255) / 256, T);
    k_combine<<<grid, 256, 0, st>>>(yacc, sh, gates, pos, k, H, (__nv_bfloat162*)y);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
