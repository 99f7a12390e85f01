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

template <int KMAX, int S>
__global__ void __launch_bounds__(256) k_route(const float* __restrict__ logits, int T, int E, int k,
                                               int32_t* __restrict__ topk_idx,
                                               float* __restrict__ gates) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* row = logits + (size_t)t * E;
    // lane l holds logits l, l+32, ... (S slots, E <= 32*S) in registers
    float val[S];
    uint32_t avail = 0u;
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int id = lane + 32 * s;
        val[s] = id < E ? __ldg(row + id) : 0.0f;
        if (id < E) avail |= 1u << s;
    }

    float sel_val[KMAX];
    int sel_id[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j >= k) break;
        // lane-local best among still-available slots
        float bv = 0.0f;
        int bi = -1;
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const int id = lane + 32 * s;
            if (((avail >> s) & 1u) && (bi < 0 || ranks_above(val[s], id, bv, bi))) {
                bv = val[s];
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
