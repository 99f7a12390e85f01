// Router top-k and renormalised gates: one warp per token.
//
// Each token picks the k largest of its E logits ("DeepSeek V4 Flash on 8x
// R9600D", model facts: 256 routed experts, 6 active per token).  Softmax is
// monotone, so the selection runs on the logits; the gates are the softmax
// renormalised over the chosen experts.  Lane l owns logits l, l+32, ...;
// each of the k rounds is a warp arg-max (ties to the lower id, NaN last)
// followed by clearing the winner's bit in its owner's mask.
#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

// a (id ia) ranks above b (id ib): larger value, then lower id; NaN last.
__device__ __forceinline__ bool ranks_above(float a, int ia, float b, int ib) {
    const bool na = a != a, nb = b != b;
    if (na || nb) return (na && nb) ? ia < ib : nb;
    if (a != b) return a > b;
    return ia < ib;
}

template <int KMAX>
__global__ void __launch_bounds__(256) k_route(const float* __restrict__ logits, int T, int E, int k,
                                               int32_t* __restrict__ topk_idx,
                                               float* __restrict__ gates) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + (size_t)t * E;
    const int per_lane = (E + 31) >> 5;  // <= 32 because E <= 1024
    uint32_t avail = per_lane >= 32 ? 0xffffffffu : ((1u << per_lane) - 1u);
    // drop slots past E
    for (int s = 0; s < per_lane; ++s)
        if (lane + 32 * s >= E) avail &= ~(1u << s);

    float sel_val[KMAX];
    int sel_id[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j >= k) break;
        // lane-local best among still-available slots
        float bv = 0.0f;
        int bi = -1;
        for (uint32_t m = avail; m; m &= m - 1) {
            const int s = __ffs(m) - 1;
            const int id = lane + 32 * s;
            const float v = __ldg(row + id);
            if (bi < 0 || ranks_above(v, id, bv, bi)) {
                bv = v;
                bi = id;
            }
        }
        // warp arg-max; lanes without a candidate carry id -1
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (oi >= 0 && (bi < 0 || ranks_above(ov, oi, bv, bi))) {
                bv = ov;
                bi = oi;
            }
        }
        sel_val[j] = bv;
        sel_id[j] = bi;
        if ((bi & 31) == lane) avail &= ~(1u << (bi >> 5));
    }
    // gates: exp(l_j - l_0) / sum, fp32, slot order
    if (lane == 0) {
        float e[KMAX];
        float den = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= k) break;
            e[j] = layer_exp(__fsub_rn(sel_val[j], sel_val[0]));
            den = __fadd_rn(den, e[j]);
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j >= k) break;
            topk_idx[(size_t)t * k + j] = sel_id[j];
            gates[(size_t)t * k + j] = __fdiv_rn(e[j], den);
        }
    }
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* gates,
                         cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int warps = 8;
    dim3 grid((T + warps - 1) / warps);
    const cudaError_t e =
        k <= 8 ? launch_pdl(k_route<8>, grid, dim3(warps * 32), 0, st, logits, T, E, k, topk_idx, gates)
               : launch_pdl(k_route<16>, grid, dim3(warps * 32), 0, st, logits, T, E, k, topk_idx, gates);
    count_launches(1);
    return e;
}

}  // namespace moe
