// Router projection: logits[t, e] = sum_h x[t, h] * Wr[e, h] + b[e].
//
// The step in front of the routed layer ("DeepSeek V4 Flash on 8x R9600D",
// model facts: 256 routed experts, 6 active per token): one logit per routed
// expert, a plain linear map of the bf16 activations with fp32 router weights.
// The layer itself takes logits as an input; this kernel produces them.
//
// A dense fp32 contraction [T, H] x [E, H]^T on CUDA cores (fp32 operands: the
// tensor cores' fp32-input path would round the weights to tf32).  CTA tile of
// 64 tokens x 64 experts, 32 inputs per step staged through shared memory
// (x widened from bf16 exactly); each of the 256 threads owns 4 x 4 outputs
// (tokens ty + 16i, experts tx + 16j) and accumulates them with fused
// multiply-adds in ascending h.  Error: |logit - S| <= gamma_(H+1) * sum_h
// |x_h Wr_h| + one rounding of the bias addition (gamma_n = n u / (1 - n u),
// u = 2^-24), whatever the summation order.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

constexpr int RT_T = 64, RT_E = 64, RT_K = 32;

__global__ void __launch_bounds__(256)
    k_router_logits(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr,
                    const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits) {
    pdl_begin();
    __shared__ float xs[RT_K][RT_T + 1];
    __shared__ float ws[RT_K][RT_E + 1];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int t0 = blockIdx.y * RT_T, e0 = blockIdx.x * RT_E;
    // loader: row tid / 4 of the tile, inputs (tid % 4) * 8 .. + 7 of the step
    const int lr = tid >> 2, lk = (tid & 3) * 8;
    const bool x_ok = t0 + lr < T, w_ok = e0 + lr < E;
    const __nv_bfloat16* xrow = x + (size_t)(x_ok ? t0 + lr : 0) * H + lk;
    const float* wrow = wr + (size_t)(w_ok ? e0 + lr : 0) * H + lk;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < H; k0 += RT_K) {
        uint4 xv = make_uint4(0u, 0u, 0u, 0u);
        float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
        if (x_ok) xv = __ldg(reinterpret_cast<const uint4*>(xrow + k0));
        if (w_ok) {
            w0 = __ldg(reinterpret_cast<const float4*>(wrow + k0));
            w1 = __ldg(reinterpret_cast<const float4*>(wrow + k0 + 4));
        }
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xs[lk + 2 * j][lr] = __uint_as_float(xw[j] << 16);             // bf16 -> fp32, exact
            xs[lk + 2 * j + 1][lr] = __uint_as_float(xw[j] & 0xffff0000u);
        }
        ws[lk + 0][lr] = w0.x;
        ws[lk + 1][lr] = w0.y;
        ws[lk + 2][lr] = w0.z;
        ws[lk + 3][lr] = w0.w;
        ws[lk + 4][lr] = w1.x;
        ws[lk + 5][lr] = w1.y;
        ws[lk + 6][lr] = w1.z;
        ws[lk + 7][lr] = w1.w;
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < RT_K; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = ws[kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + ty + 16 * i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tx + 16 * j;
            if (e < E) logits[(size_t)t * E + e] = bias ? __fadd_rn(acc[i][j], __ldg(bias + e)) : acc[i][j];
        }
    }
}

// Few tokens (decode): the tiled kernel above would run a handful of CTAs.
// Instead a warp computes one expert's logits for all T <= kRouterSmallT
// tokens: lane l walks h = 8 l, 8 l + 256, ... , loading 8 router weights
// (two float4) and, for every token, 8 bf16 inputs (one uint4, from L1/L2:
// the T rows are shared by every warp), accumulating per token with fused
// multiply-adds; the per-lane partial sums are then added across the warp.
// The same summation bound holds (any order).  The router weights, the
// dominant bytes, are read once, coalesced.
constexpr int kRouterSmallT = 16;

template <int TMAX>
__global__ void __launch_bounds__(256)
    k_router_logits_small(const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr,
                          const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits) {
    pdl_begin();
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= E) return;
    float acc[TMAX];
#pragma unroll
    for (int t = 0; t < TMAX; ++t) acc[t] = 0.0f;
    const float* wrow = wr + (size_t)e * H;
    for (int h = 8 * lane; h < H; h += 256) {
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(wrow + h));
        const float4 w1 = __ldg(reinterpret_cast<const float4*>(wrow + h + 4));
        const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
            if (t < T) {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * H + h));
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[t] = __fmaf_rn(__uint_as_float(xw[j] << 16), w[2 * j], acc[t]);          // bf16 -> fp32, exact
                    acc[t] = __fmaf_rn(__uint_as_float(xw[j] & 0xffff0000u), w[2 * j + 1], acc[t]);
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
        if (t < T) {
            float v = acc[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) logits[(size_t)t * E + e] = bias ? __fadd_rn(v, __ldg(bias + e)) : v;
        }
    }
}

cudaError_t launch_router_logits(const void* x, const float* wr, const float* bias, int T, int H, int E,
                                 float* logits, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (T <= kRouterSmallT) {
        const cudaError_t e = launch_pdl(k_router_logits_small<kRouterSmallT>, dim3((unsigned)((E + 7) / 8)),
                                         dim3(256), 0, st, (const __nv_bfloat16*)x, wr, bias, T, H, E, logits);
        count_launches(1);
        return e;
    }
    const dim3 grid((unsigned)((E + RT_E - 1) / RT_E), (unsigned)((T + RT_T - 1) / RT_T));
    const cudaError_t e = launch_pdl(k_router_logits, grid, dim3(256), 0, st, (const __nv_bfloat16*)x, wr, bias,
                                     T, H, E, logits);
    count_launches(1);
    return e;
}

}  // namespace moe
