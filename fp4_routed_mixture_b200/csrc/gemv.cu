// Streaming grouped GEMM for the decode regime (few tokens per expert).
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) drives its decode expert
// GEMMs from packed FP4 weights and INT8 activations with integer
// dot-product instructions, and names memory bandwidth and low M as the
// limits.  On B200 the same regime is HBM-bound: every touched expert's FP4
// weights are read exactly once, with 128-bit coalesced loads, while the few
// token rows of that expert are reused from L1.
//
// Work: for every expert e with M_e > 0, units (tile of 32 weight rows, group
// of up to kGroup tokens); each unit is K/128 items of 4 scale blocks.  The
// flat item range is split evenly over all warps of the grid (stream-K), so
// the load is balanced to within one item whatever the expert counts are.
// Lane l of a warp owns weight row 32*tile + l and the full dot products of
// that row with the group's token rows:
//   * a 16-byte code load gives the lane one 32-element block (one scale);
//   * nibbles become bytes 2*e2m1 + 12 in [0, 24] through two byte
//     permutes (positive and negative code tables) and an OR;
//   * __dp4a against the int8 activation bytes, started from -12 * (sum of
//     the block's activation codes), gives the exact integer block sum;
//   * block sums are scaled by 2^(S-128) and accumulated in fp64, exact for
//     every realistic scale spread (each term is an integer multiple of the
//     row's smallest scale).
// A warp's partial sums are added to fp64 accumulators with atomicAdd; as all
// partial sums are exact, the result is independent of the order.
#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

constexpr int kGroup = 8;        // token rows per unit
constexpr int kGemvWarps = 8;    // warps per CTA
constexpr int kGroupBytes = 2176;  // 4 scale blocks of 32 rows: 128 B scales + 4 x 512 B codes

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// 8 E2M1 codes (one 32-bit word, element j in nibble j) -> two words of
// unsigned bytes 2*e2m1 + 12.  prmt's selector nibble: bits 0-2 pick a table
// byte, bit 3 (the code's sign) replicates that byte's sign bit instead, which
// is 0 for every table byte.  So the positive table answers for sign 0 codes,
// the negative table (selected with the sign bit flipped) for sign 1 codes,
// and the other table returns 0.
__device__ __forceinline__ void decode8(uint32_t w, uint32_t& lo, uint32_t& hi) {
    constexpr uint32_t kPos0 = 0x0F0E0D0Cu, kPos1 = 0x18141210u;  // 12 + {0,1,2,3,4,6,8,12}
    constexpr uint32_t kNeg0 = 0x090A0B0Cu, kNeg1 = 0x00040608u;  // 12 - {0,1,2,3,4,6,8,12}
    const uint32_t wf = w ^ 0x88888888u;
    lo = prmt(kPos0, kPos1, w) | prmt(kNeg0, kNeg1, wf);
    hi = prmt(kPos0, kPos1, w >> 16) | prmt(kNeg0, kNeg1, wf >> 16);
}

__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

struct GemvArgs {
    const uint8_t* w;          // matrix region of the packed buffer
    size_t expert_bytes;
    int K;                     // inputs per weight row
    int N;                     // weight rows per expert (= output columns)
    const int8_t* act;         // activation codes, rows of K bytes
    const int32_t* act_init;   // rows of K/32 block terms
    const int32_t* perm;       // sorted row -> pair id
    int k_div;                 // >0: activation row = perm[i] / k_div; 0: = i
    const int32_t* offsets;    // [E+1]
    const int32_t* unit_off;   // [E+1] exclusive scan of units per expert
    int E;
    double* out;               // [P, N] fp64 accumulators, zeroed
    const int32_t* flag;       // device error word: a layout mismatch stops the kernel
};

__global__ void __launch_bounds__(kGemvWarps * 32) k_gemv(GemvArgs a) {
    const int lane = threadIdx.x & 31;
    // packed weights built for other dims may be smaller than the offsets used here
    if (*(volatile const int32_t*)a.flag & FLAG_LAYOUT) return;
    const long long gw = (long long)blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
    const long long nw = (long long)gridDim.x * kGemvWarps;
    const int KG = a.K / 128;
    const long long U = a.unit_off[a.E];
    const long long W = U * KG;
    const long long it1 = W * (gw + 1) / nw;
    long long it = W * gw / nw;
    while (it < it1) {
        const int unit = (int)(it / KG);
        const int kg0 = (int)(it % KG);
        const long long rem = it1 - it;
        const int kg1 = rem < (long long)(KG - kg0) ? kg0 + (int)rem : KG;
        // expert of this unit: last e with unit_off[e] <= unit
        int lo = 0, hi = a.E;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(a.unit_off + mid) <= unit) lo = mid; else hi = mid;
        }
        const int e = lo;
        const int r0 = __ldg(a.offsets + e), r1 = __ldg(a.offsets + e + 1);
        const int ngroups = (r1 - r0 + kGroup - 1) / kGroup;
        const int local = unit - __ldg(a.unit_off + e);
        const int tile = local / ngroups;
        const int i0 = r0 + (local % ngroups) * kGroup;
        const int mc = min(kGroup, r1 - i0);
        int arow[kGroup];
#pragma unroll
        for (int m = 0; m < kGroup; ++m) {
            const int i = i0 + min(m, mc - 1);
            arow[m] = a.k_div ? __ldg(a.perm + i) / a.k_div : i;
        }
        const uint8_t* tb = a.w + (size_t)e * a.expert_bytes + (size_t)tile * KG * kGroupBytes;
        double acc[kGroup];
#pragma unroll
        for (int m = 0; m < kGroup; ++m) acc[m] = 0.0;
        for (int kg = kg0; kg < kg1; ++kg) {
            const uint8_t* gb = tb + (size_t)kg * kGroupBytes;
            const uint32_t sw = ldg_u32(gb + lane * 4);
            uint4 c[4];
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) c[bb] = ldg_stream(gb + 128 + bb * 512 + lane * 16);
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const double sc = pow2_scale_minus128((sw >> (8 * bb)) & 0xffu);
                uint32_t v[8];
                decode8(c[bb].x, v[0], v[1]);
                decode8(c[bb].y, v[2], v[3]);
                decode8(c[bb].z, v[4], v[5]);
                decode8(c[bb].w, v[6], v[7]);
                const int blk = kg * 4 + bb;
#pragma unroll
                for (int m = 0; m < kGroup; ++m) {
                    if (m < mc) {
                        const uint4* xp = reinterpret_cast<const uint4*>(a.act + (size_t)arow[m] * a.K +
                                                                         blk * 32);
                        const uint4 x0 = __ldg(xp), x1 = __ldg(xp + 1);
                        int d = __ldg(a.act_init + (size_t)arow[m] * (a.K / 32) + blk);
                        d = __dp4a((int)v[0], (int)x0.x, d);
                        d = __dp4a((int)v[1], (int)x0.y, d);
                        d = __dp4a((int)v[2], (int)x0.z, d);
                        d = __dp4a((int)v[3], (int)x0.w, d);
                        d = __dp4a((int)v[4], (int)x1.x, d);
                        d = __dp4a((int)v[5], (int)x1.y, d);
                        d = __dp4a((int)v[6], (int)x1.z, d);
                        d = __dp4a((int)v[7], (int)x1.w, d);
                        acc[m] = __fma_rn((double)d, sc, acc[m]);
                    }
                }
            }
        }
        const int n = tile * 32 + lane;
#pragma unroll
        for (int m = 0; m < kGroup; ++m)
            if (m < mc) atomicAdd(a.out + (size_t)(i0 + m) * a.N + n, acc[m]);
        it += kg1 - kg0;
    }
}

// Units per expert for both matrices and their exclusive scans (one warp;
// lane l owns a contiguous slice of experts).
__global__ void k_plan(const int32_t* __restrict__ offsets, int E, int tiles1, int tiles2,
                       int32_t* __restrict__ unit_off1, int32_t* __restrict__ unit_off2) {
    const int lane = threadIdx.x;
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int s1 = 0, s2 = 0;
    for (int e = e0; e < e1; ++e) {
        const int g = (offsets[e + 1] - offsets[e] + kGroup - 1) / kGroup;
        s1 += g * tiles1;
        s2 += g * tiles2;
    }
    int x1 = s1, x2 = s2;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y1 = __shfl_up_sync(0xffffffffu, x1, o), y2 = __shfl_up_sync(0xffffffffu, x2, o);
        if (lane >= o) {
            x1 += y1;
            x2 += y2;
        }
    }
    int r1 = x1 - s1, r2 = x2 - s2;  // exclusive prefix
    for (int e = e0; e < e1; ++e) {
        unit_off1[e] = r1;
        unit_off2[e] = r2;
        const int g = (offsets[e + 1] - offsets[e] + kGroup - 1) / kGroup;
        r1 += g * tiles1;
        r2 += g * tiles2;
    }
    if (lane == 31) {
        unit_off1[E] = x1;
        unit_off2[E] = x2;
    }
}

static int gemv_grid() {
    static int grid = 0;
    if (!grid) {
        int dev = 0, sms = 0, per_sm = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv, kGemvWarps * 32, 0);
        grid = sms * (per_sm > 0 ? per_sm : 1);
    }
    return grid;
}

cudaError_t launch_plan(const int32_t* offsets, int E, int tiles1, int tiles2, int32_t* unit_off1,
                        int32_t* unit_off2, cudaStream_t st) {
    k_plan<<<1, 32, 0, st>>>(offsets, E, tiles1, tiles2, unit_off1, unit_off2);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_gemv(const uint8_t* w, size_t expert_bytes, int K, int N, const int8_t* act,
                        const int32_t* act_init, const int32_t* perm, int k_div,
                        const int32_t* offsets, const int32_t* unit_off, int E, double* out,
                        const int32_t* flag, cudaStream_t st) {
    GemvArgs a{w, expert_bytes, K, N, act, act_init, perm, k_div, offsets, unit_off, E, out, flag};
    k_gemv<<<gemv_grid(), kGemvWarps * 32, 0, st>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
