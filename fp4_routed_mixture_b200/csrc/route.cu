// Router top-k and renormalised gates: one warp per token (route_token in
// steps.cuh: the k largest logits, ties to the lower id, NaN last; gates are
// the softmax renormalised over the chosen experts).
#include "steps.cuh"

namespace moe {

template <int KMAX, int S>
__global__ void __launch_bounds__(256) k_route(const float* __restrict__ logits, int T, int E, int k,
                                               int32_t* __restrict__ topk_idx,
                                               float* __restrict__ gates) {
    pdl_begin();
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    route_token<KMAX, S>(logits + (size_t)t * E, E, k, topk_idx + (size_t)t * k, gates + (size_t)t * k, nullptr);
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* gates,
                         cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int warps = 8;
    dim3 grid((T + warps - 1) / warps);
    cudaError_t e;
    if (E <= 256)
        e = k <= 8 ? launch_pdl(k_route<8, 8>, grid, dim3(warps * 32), 0, st, logits, T, E, k, topk_idx, gates)
                   : launch_pdl(k_route<16, 8>, grid, dim3(warps * 32), 0, st, logits, T, E, k, topk_idx, gates);
    else
        e = k <= 8 ? launch_pdl(k_route<8, 32>, grid, dim3(warps * 32), 0, st, logits, T, E, k, topk_idx, gates)
                   : launch_pdl(k_route<16, 32>, grid, dim3(warps * 32), 0, st, logits, T, E, k, topk_idx, gates);
    count_launches(1);
    return e;
}

}  // namespace moe
