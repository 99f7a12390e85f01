// INT8 activation quantisation ("DeepSeek-V4-Flash on AMD gfx90a", abstract:
// INT8 activations feeding the packed-FP4 expert GEMMs).
//
//   k_xquant        x [T,H] bf16 -> xq [T,H] int8, sx [T], xinit [T,H/32], and
//                   (tensor-core path) the x digit planes in token order; also
//                   checks the packed header and clears the call's error word
//   k_hquant        h of every sorted row (SwiGLU of the streaming GEMM's fp64
//                   sums, or h from the tensor-core epilogue) -> hq, sh, hinit,
//                   or the W2 digit planes for tensor-core rows
//   k_quant_rows    fp32 rows -> int8 + scale (stage entry point)
//
// Rule for every row: a = max|v| (exact), s = fp32(a/127) by IEEE division,
// q = clamp(rne(fp32(v/s)), -127, 127), and q = 0, s = 0 for an all-zero row.
// xinit/hinit hold -12 * (sum of the 32 codes of each K block): the streaming
// GEMM decodes weight nibbles to 2*e2m1 + 12 (an unsigned byte), so this term
// cancels the +12 bias of every block's integer dot product.  The per-token
// body of the x quant is xquant_row (steps.cuh).
#include "steps.cuh"

namespace moe {

// One CTA per token (xquant_row).  It is also the first kernel of
// moe_forward: thread 0 of CTA 0 clears the call's device error word and sets
// FLAG_LAYOUT when the packed buffer was built for other dims (no other CTA of
// this kernel touches the word).  The tensor-core GEMM's plane writer copies
// the token-order digit planes (tplanes) into sorted-row order.
__global__ void __launch_bounds__(kQThreads)
    k_xquant(const __nv_bfloat16* __restrict__ x, int T, int H, int8_t* __restrict__ xq,
             float* __restrict__ sx, int32_t* __restrict__ xinit, uint8_t* __restrict__ tplanes,
             int8_t* __restrict__ dbg_xq, float* __restrict__ dbg_sx, const void* __restrict__ packed, int I,
             int E, int32_t* flag) {
    pdl_begin();
    if (blockIdx.x == 0 && threadIdx.x == 0) *flag = packed_header_ok(packed, H, I, E) ? 0 : FLAG_LAYOUT;
    __shared__ float red[33];
    __shared__ uint16_t lut[256];
    xquant_row(x, blockIdx.x, H, xq, sx, xinit, tplanes, dbg_xq, dbg_sx, red, lut);
}

// R threads per sorted row (R = 32: a warp per row, for many rows; R = 256:
// a CTA per row, for few), grid-stride over rows: the row's h values and |h|
// maximum, then its INT8 codes.  Rows of experts on the streaming GEMM arrive
// as exact fp64 sums of the W1 product (gate and up):
// G = fp32(fp64(sx[t]) * sum), h = SwiGLU(g, u) is formed here and parked in
// hbuf; rows of experts on the tensor-core GEMM arrive as h itself in hbuf
// (formed in that GEMM's epilogue).  Pass 1 reads the row and reduces the
// maximum, pass 2 reads it again (each thread its own elements, from cache)
// and quantises: streaming rows get hq and the block sums hinit their GEMM
// needs, tensor-core rows get the digit planes of the W2 tensor-core GEMM
// written directly (plane row plane_row[i]).  Thread l of a row holds the
// elements 4*(l + R*g) .. +3 in step g; 8 consecutive threads cover one
// 32-input chunk.  KEEP > 0 (rows of at most 4*R*KEEP elements): pass 1 keeps
// the values in registers for pass 2 instead of reading them again.
template <int R, int KEEP>
__global__ void __launch_bounds__(kQThreads)
    k_hquant(const double* __restrict__ gacc, float* __restrict__ hbuf, const float* __restrict__ sx,
             const int32_t* __restrict__ perm, const int32_t* __restrict__ plane_row, int plane_rows,
             int stream_rows, uint8_t* __restrict__ planes, int P, int k, int I, int8_t* __restrict__ hq,
             float* __restrict__ sh, int32_t* __restrict__ hinit, int8_t* __restrict__ dbg_hq,
             float* __restrict__ dbg_sh, int32_t* flag) {
    static_assert(R == 32 || R == kQThreads, "a warp or a CTA per row");
    float4 keep[KEEP > 0 ? KEEP : 1];
    __shared__ uint16_t lut[256];
    __shared__ float red[33];
    for (int v = threadIdx.x; v < 256; v += blockDim.x) lut[v] = (uint16_t)digit_codes((int)(int8_t)v);
    __syncthreads();
    const int l = threadIdx.x % R;
    const int rows_per_cta = kQThreads / R;
    const int steps = I / (4 * R);          // I % 128 == 0; for R = 256 also I % 1024 == 0 (checked by the launcher)
    // A row's slot, pair and x scale come from the plan, sort and x quant,
    // launches before the W1 GEMM in front of this one (which had completed
    // when that GEMM passed its own wait): the first row's are read before
    // waiting on the GEMM, whose output (the W1 sums or h) is read after.
    auto row_slot = [&](int i) { return i < P ? plane_row[i] : kNoRow; };
    int pre_slot = row_slot(blockIdx.x * rows_per_cta + (int)threadIdx.x / R), pre_p = 0;
    float pre_sx = 0.0f;
    {
        const int i = blockIdx.x * rows_per_cta + (int)threadIdx.x / R;
        if (i < P && pre_slot != kNoRow) {
            pre_p = checked_index(perm[i], P, flag);
            if (pre_slot < 0) pre_sx = sx[pre_p / k];
        }
    }
    pdl_begin();
    for (int i0 = blockIdx.x * rows_per_cta; i0 < P; i0 += gridDim.x * rows_per_cta) {
        const bool first = i0 == (int)blockIdx.x * rows_per_cta;
        const int i = i0 + (int)threadIdx.x / R;
        // (R = 256: always in range; a row's R threads take the same branches)
        const int slot = first ? pre_slot : row_slot(i);
        const bool tc = slot >= 0;
        const int srow = ~slot;              // streaming row (slot < 0)
        const bool slot_ok = tc ? slot < plane_rows : (slot != kNoRow && srow < stream_rows);
        if (i < P && !slot_ok && threadIdx.x % R == 0) raise_flag(flag, FLAG_BOUNDS);
        const bool row_ok = i < P && slot_ok;
        float a = 0.0f;
        int p = 0;
        if (row_ok) p = first ? pre_p : checked_index(perm[i], P, flag);
        float4* hr = reinterpret_cast<float4*>(hbuf + (size_t)(row_ok ? i : 0) * I);
        // KEEP > 0 and the row fits: pass 1 leaves the row in registers
        const bool use_keep = KEEP > 0 && steps <= KEEP;
        if (row_ok && tc) {
            if (use_keep) {
#pragma unroll
                for (int g = 0; g < (KEEP > 0 ? KEEP : 1); ++g)
                    if (g < steps) {
                        keep[g] = hr[g * R + l];
                        a = fmaxf(fmaxf(a, fabsf(keep[g].x)), fmaxf(fmaxf(fabsf(keep[g].y), fabsf(keep[g].z)),
                                                                   fabsf(keep[g].w)));
                    }
            } else {
#pragma unroll 4
                for (int g = 0; g < steps; ++g) {
                    const float4 v = hr[g * R + l];
                    a = fmaxf(fmaxf(a, fabsf(v.x)), fmaxf(fmaxf(fabsf(v.y), fabsf(v.z)), fabsf(v.w)));
                }
            }
        } else if (row_ok) {
            const double s = (double)(first ? pre_sx : sx[p / k]);
            const double* gr = gacc + (size_t)srow * 2 * I;
            for (int g = 0; g < steps; ++g) {
                const int e0 = 4 * (g * R + l);
                float hv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float gv = (float)__dmul_rn(s, gr[e0 + u]);
                    const float uv = (float)__dmul_rn(s, gr[I + e0 + u]);
                    hv[u] = swiglu(gv, uv);
                    a = fmaxf(a, fabsf(hv[u]));
                }
                const float4 h4 = make_float4(hv[0], hv[1], hv[2], hv[3]);
                if (use_keep) {
#pragma unroll
                    for (int u = 0; u < (KEEP > 0 ? KEEP : 1); ++u)
                        if (u == g) keep[u] = h4;
                } else {
                    hr[g * R + l] = h4;  // read back by this thread
                }
            }
        }
        if (R == 32)
            a = warp_max(a);
        else
            a = block_max(a, red);
        if (!row_ok) continue;  // (R = 32 only: whole warps skip together)
        const float sc = quant_scale(a);
        if (l == 0) {
            sh[i] = sc;
            if (dbg_sh) dbg_sh[i] = sc;
        }
        const int pr = tc ? slot : -1;
#pragma unroll(KEEP > 0 ? KEEP : 4)
        for (int g = 0; g < steps; ++g) {
            const int e0 = 4 * (g * R + l);
            float4 v;
            if (use_keep) {
                // (the loop is unrolled KEEP times, so the index is a constant)
#pragma unroll
                for (int u = 0; u < (KEEP > 0 ? KEEP : 1); ++u)
                    if (u == g) v = keep[u];
            } else {
                v = hr[g * R + l];
            }
            const int q[4] = {quant_code(v.x, a, sc), quant_code(v.y, a, sc), quant_code(v.z, a, sc),
                              quant_code(v.w, a, sc)};
            const uint32_t packed = (uint32_t)(q[0] & 0xff) | (uint32_t)(q[1] & 0xff) << 8 |
                                    (uint32_t)(q[2] & 0xff) << 16 | (uint32_t)(q[3] & 0xff) << 24;
            if (dbg_hq) *reinterpret_cast<uint32_t*>(dbg_hq + (size_t)i * I + e0) = packed;
            if (!tc) {
                *reinterpret_cast<uint32_t*>(hq + (size_t)srow * I + e0) = packed;
                int bsum = q[0] + q[1] + q[2] + q[3];
                bsum += __shfl_xor_sync(0xffffffffu, bsum, 1);
                bsum += __shfl_xor_sync(0xffffffffu, bsum, 2);
                bsum += __shfl_xor_sync(0xffffffffu, bsum, 4);
                if ((l & 7) == 0) hinit[(size_t)srow * (I / 32) + (e0 >> 5)] = -12 * bsum;
            } else if (pr >= 0) {
                // 4 codes = 16 bits of each plane's 16-byte piece of chunk e0/32
                uint32_t d[3] = {0u, 0u, 0u};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t t = lut[q[u] & 0xff];
                    d[0] |= (t & 0xFu) << (4 * u);
                    d[1] |= ((t >> 4) & 0xFu) << (4 * u);
                    d[2] |= (t >> 8) << (4 * u);
                }
                const int st = e0 >> 7, cc = (e0 >> 5) & 3;
                uint8_t* dst = planes + ((size_t)st * (plane_rows / 8) + (pr >> 3)) * kPlaneGroupBytes +
                               cc * 128 + (pr & 7) * 16 + ((e0 & 31) >> 2) * 2;
#pragma unroll
                for (int pl = 0; pl < 3; ++pl) *reinterpret_cast<uint16_t*>(dst + pl * 512) = (uint16_t)d[pl];
            }
        }
    }
}


__global__ void __launch_bounds__(kQThreads)
    k_quant_rows(const float* __restrict__ v, int cols, int8_t* __restrict__ q, float* __restrict__ s) {
    __shared__ float red[33];
    const int r = blockIdx.x;
    const float* row = v + (size_t)r * cols;
    float a = 0.0f;
    for (int c = threadIdx.x; c < cols; c += blockDim.x) a = fmaxf(a, fabsf(row[c]));
    a = block_max(a, red);
    const float sc = quant_scale(a);
    if (threadIdx.x == 0) s[r] = sc;
    for (int c = threadIdx.x; c < cols; c += blockDim.x)
        q[(size_t)r * cols + c] = (int8_t)quant_code(row[c], a, sc);
}

__global__ void k_exp(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        y[i] = layer_exp(x[i]);
}

__global__ void k_swiglu(const float* __restrict__ g, const float* __restrict__ u,
                         float* __restrict__ h, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        h[i] = swiglu(g[i], u[i]);
}

cudaError_t launch_exp(const float* x, float* y, int64_t n, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    const int grid = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
    k_exp<<<grid, 256, 0, st>>>(x, y, n);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_swiglu(const float* g, const float* u, float* h, int64_t n, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    const int grid = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
    k_swiglu<<<grid, 256, 0, st>>>(g, u, h, n);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_xquant(const void* x, int T, int H, int8_t* xq, float* sx, int32_t* xinit,
                          uint8_t* tplanes, int8_t* dbg_xq, float* dbg_sx, const void* packed, int I, int E,
                          int32_t* flag, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const cudaError_t e = launch_pdl(k_xquant, dim3(T), dim3(kQThreads), 0, st, (const __nv_bfloat16*)x, T, H,
                                     xq, sx, xinit, tplanes, dbg_xq, dbg_sx, packed, I, E, flag);
    count_launches(1);
    return e;
}

cudaError_t launch_hquant(const double* gacc, float* hbuf, const float* sx, const int32_t* perm,
                          const int32_t* plane_row, int plane_rows, int stream_rows, uint8_t* planes, int P, int k,
                          int I, int8_t* hq, float* sh, int32_t* hinit, int8_t* dbg_hq, float* dbg_sh, int32_t* flag,
                          cudaStream_t st) {
    if (P == 0) return cudaSuccess;
    // few rows (decode): a CTA per row keeps every row's chain short; many
    // rows (prefill): a warp per row needs no block barriers
    cudaError_t e;
    if (P < 4096 && I % (4 * kQThreads) == 0) {
        // (a thread holds 4 * I / (4 * kQThreads) values: at most 4 float4 up to I = 4096)
        e = launch_pdl(k_hquant<kQThreads, 4>, dim3(std::min(P, 148 * 8)), dim3(kQThreads), 0, st, gacc, hbuf, sx,
                       perm, plane_row, plane_rows, stream_rows, planes, P, k, I, hq, sh, hinit, dbg_hq, dbg_sh,
                       flag);
    } else {
        const int warps = kQThreads / 32;
        const int grid = std::min((P + warps - 1) / warps, 148 * 8);
        // (keeping a row in registers between the passes, k_hquant<32, 16>,
        // measured slower: 112 registers halve the rows in flight)
        e = launch_pdl(k_hquant<32, 0>, dim3(grid), dim3(kQThreads), 0, st, gacc, hbuf, sx, perm, plane_row,
                       plane_rows, stream_rows, planes, P, k, I, hq, sh, hinit, dbg_hq, dbg_sh, flag);
    }
    count_launches(1);
    return e;
}


cudaError_t launch_quant_rows(const float* v, int rows, int cols, int8_t* q, float* s,
                              cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    k_quant_rows<<<rows, kQThreads, 0, st>>>(v, cols, q, s);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
