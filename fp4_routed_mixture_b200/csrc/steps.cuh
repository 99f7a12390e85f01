// Device bodies of the steps before the first expert GEMM -- route, sort,
// x quant and plan -- shared by each step's own kernel and by the fused
// launch that runs all four for decode-size calls (front.cu).
#pragma once
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "moe_common.cuh"

namespace moe {

// ---- route -------------------------------------------------------------------
// Each token picks the k largest of its E logits ("DeepSeek V4 Flash on 8x
// R9600D", model facts: 256 routed experts, 6 active per token).  Softmax is
// monotone, so the selection runs on the logits; the gates are the softmax
// renormalised over the chosen experts.

// a (id ia) ranks above b (id ib): larger value, then lower id; NaN last.
__device__ __forceinline__ bool ranks_above(float a, int ia, float b, int ib) {
    const bool na = a != a, nb = b != b;
    if (na || nb) return (na && nb) ? ia < ib : nb;
    if (a != b) return a > b;
    return ia < ib;
}

// One warp routes one token: row holds its E logits (E <= 32*S), k <= KMAX
// <= 32; the k chosen ids and gates go to idx_out[0..k) and gates_out[0..k),
// and the ids also to idx_copy[0..k) when it is not NULL.  Lane l owns logits l, l+32, ... in
// registers; each of the k rounds is a warp arg-max (ties to the lower id,
// NaN last) followed by clearing the winner's bit in its owner's mask.
template <int KMAX, int S>
__device__ __forceinline__ void route_token(const float* __restrict__ row, int E, int k,
                                            int32_t* __restrict__ idx_out, float* __restrict__ gates_out,
                                            int32_t* idx_copy) {
    const int lane = threadIdx.x & 31;
    float val[S];
    uint32_t avail = 0u;
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int id = lane + 32 * s;
        val[s] = id < E ? __ldg(row + id) : 0.0f;
        if (id < E) avail |= 1u << s;
    }

    // k rounds; round j's winner is kept by lane j (the loop body is emitted
    // once: this code runs once per layer call, with a cold instruction cache)
    float top = 0.0f, my_val = 0.0f;
    int my_id = -1;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
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
        if (j == 0) top = bv;
        if (lane == j) {
            my_val = bv;
            my_id = bi;
        }
        if ((bi & 31) == lane) avail &= ~(1u << (bi >> 5));
    }
    // gates: lane j < k forms exp(l_j - l_0) (all lanes at once); the
    // denominator is summed in slot order, then lane j divides
    const float e = layer_exp(__fsub_rn(my_val, top));
    float den = 0.0f;
#pragma unroll 1
    for (int j = 0; j < k; ++j) den = __fadd_rn(den, __shfl_sync(0xffffffffu, e, j));
    if (lane < k) {
        idx_out[lane] = my_id;
        gates_out[lane] = __fdiv_rn(e, den);
        if (idx_copy) idx_copy[lane] = my_id;
    }
}

// ---- sort ------------------------------------------------------------------------
constexpr int kSortChunk = 1024;
constexpr int kSortThreads = 256;

__device__ __forceinline__ bool valid_expert(int e, int E) { return (unsigned)e < (unsigned)E; }

// Exclusive scan of vals[0..E) in place (blockDim == kSortThreads, E <= 1024);
// returns the total.  Warp 0 scans (lane l owns a contiguous slice of at most
// 32 entries); the other warps wait at the two barriers.  `tmp` [1] is shared
// scratch for the total.
static __device__ int block_exclusive_scan(int* vals, int E, int* tmp) {
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int per = (E + 31) / 32;
        const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
        int s = 0;
        for (int e = e0; e < e1; ++e) s += vals[e];
        int x = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        int run = x - s;
        for (int e = e0; e < e1; ++e) {
            const int v = vals[e];
            vals[e] = run;
            run += v;
        }
        if (lane == 31) tmp[0] = x;
    }
    __syncthreads();
    return tmp[0];
}

// Stable scatter of pairs [p0, p1) (at most 32 x 32 of them) by one warp;
// expert_of(p) gives pair p's expert id, cursor[e] is the next free sorted
// slot of expert e and is advanced in place.  The warp first loads all of its
// expert ids (lane l holds pairs p0 + 32s + l) so the serial steps wait on no
// load.  __match_any_sync ranks equal experts inside each 32-pair step, which
// keeps the sort stable.
template <class ExpertOf>
__device__ __forceinline__ void warp_stable_scatter(ExpertOf expert_of, int p0, int p1, int E, int* cursor,
                                                    int32_t* __restrict__ perm, int32_t* __restrict__ pos) {
    const int lane = threadIdx.x & 31;
    int ids[32];
#pragma unroll
    for (int s = 0; s < 32; ++s) {
        const int p = p0 + 32 * s + lane;
        ids[s] = p < p1 ? expert_of(p) : -1;
    }
#pragma unroll
    for (int s = 0; s < 32; ++s) {
        const int base = p0 + 32 * s;
        if (base >= p1) break;
        const int p = base + lane;
        int e = ids[s];
        if (p >= p1 || !valid_expert(e, E)) e = -1 - lane;  // unique key: never grouped, never written
        const uint32_t same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & ((1u << lane) - 1u));
        const int leader = __ffs(same) - 1;
        int slot = 0;
        if (e >= 0) slot = cursor[e];  // all lanes of a group read the same value
        __syncwarp();
        if (e >= 0) {
            const int dst = slot + rank;
            perm[dst] = p;
            pos[p] = dst;
            if (lane == leader) cursor[e] = slot + __popc(same);
        }
        __syncwarp();
    }
}

// The whole sort of P <= kSortChunk pairs by one CTA of kSortThreads threads:
// histogram in shared memory, exclusive scan into offsets, stable scatter.
// hist [E] and tmp [kSortThreads + 1] are shared scratch; offs_copy (shared,
// E + 1 entries, may be NULL) receives the offsets too.  Expert ids outside
// [0, E) raise FLAG_BAD_EXPERT and are skipped.
template <class ExpertOf>
__device__ __forceinline__ void sort_cta(ExpertOf expert_of, int P, int E, int32_t* __restrict__ perm,
                                         int32_t* __restrict__ pos, int32_t* __restrict__ offsets, int* hist,
                                         int* tmp, int* offs_copy, int32_t* flag) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    bool bad = false;
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        const int e = expert_of(p);
        if (valid_expert(e, E))
            atomicAdd(&hist[e], 1);
        else
            bad = true;
    }
    if (bad) raise_flag(flag, FLAG_BAD_EXPERT);
    __syncthreads();
    const int all = block_exclusive_scan(hist, E, tmp);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        offsets[e] = hist[e];
        if (offs_copy) offs_copy[e] = hist[e];
    }
    if (threadIdx.x == 0) {
        offsets[E] = all;
        if (offs_copy) offs_copy[E] = all;
    }
    __syncthreads();
    if (threadIdx.x < 32) warp_stable_scatter(expert_of, 0, P, E, hist, perm, pos);
}

// ---- x quant -----------------------------------------------------------------------
// INT8 activation quantisation ("DeepSeek-V4-Flash on AMD gfx90a", abstract).
// Rule for every row: a = max|v| (exact), s = fp32(a/127) by IEEE division,
// q = clamp(rne(fp32(v/s)), -127, 127), and q = 0, s = 0 for an all-zero row.
constexpr int kQThreads = 256;
static_assert(kQThreads == kSortThreads, "the fused front kernel runs both with one block size");
static_assert(kSortChunk == kFrontMaxPairs, "the fused front kernel sorts one chunk");

__device__ __forceinline__ float block_max(float v, float* red) {
    v = warp_max(v);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[w] = v;
    __syncthreads();
    if (w == 0) {
        v = (lane < (int)(blockDim.x >> 5)) ? red[lane] : 0.0f;
        v = warp_max(v);
        if (lane == 0) red[32] = v;
    }
    __syncthreads();
    const float r = red[32];
    __syncthreads();
    return r;
}

// One CTA (kQThreads threads) quantises token t: x [T,H] bf16 -> xq [T,H]
// int8, sx [T], xinit [T,H/32] (-12 * the sum of each 32-input block's codes:
// the streaming GEMM decodes weight nibbles to 2*e2m1 + 12, and this term
// cancels the +12 bias of every block's integer dot product).  Each thread
// handles chunks of 8 consecutive elements.  With tplanes != NULL the token's
// codes are also written once as E2M1 digit planes in token order: per
// 32-input block b, 48 bytes at tplanes + (t*(H/32) + b)*48: plane p's 16
// bytes at +16p (element 2j of the block in the low nibble of byte j).  red
// [33] and lut [256] are shared scratch.
__device__ __forceinline__ void xquant_row(const __nv_bfloat16* __restrict__ x, int t, int H,
                                           int8_t* __restrict__ xq, float* __restrict__ sx,
                                           int32_t* __restrict__ xinit, uint8_t* __restrict__ tplanes,
                                           int8_t* __restrict__ dbg_xq, float* __restrict__ dbg_sx, float* red,
                                           uint16_t* lut) {
    if (tplanes)
        for (int v = threadIdx.x; v < 256; v += blockDim.x) lut[v] = (uint16_t)digit_codes((int)(int8_t)v);
    const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)t * H);
    const int nchunk = H / 8;
    float a = 0.0f;
    for (int c = threadIdx.x; c < nchunk; c += blockDim.x) {
        const uint4 v = __ldg(row + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            a = fmaxf(a, fabsf(__uint_as_float(w[j] << 16)));
            a = fmaxf(a, fabsf(__uint_as_float(w[j] & 0xffff0000u)));
        }
    }
    a = block_max(a, red);  // (its barriers also publish lut)
    const float s = quant_scale(a);
    if (threadIdx.x == 0) {
        sx[t] = s;
        if (dbg_sx) dbg_sx[t] = s;
    }
    // chunks are handed out round-robin, so the 4 chunks of one 32-element
    // block sit in 4 consecutive lanes of one warp (nchunk % 4 == 0)
    for (int c0 = 0; c0 < nchunk; c0 += blockDim.x) {
        const int c = c0 + threadIdx.x;
        int bsum = 0;
        if (c < nchunk) {
            const uint4 v = __ldg(row + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int q0 = quant_code(__uint_as_float(w[j] << 16), a, s);
                const int q1 = quant_code(__uint_as_float(w[j] & 0xffff0000u), a, s);
                bsum += q0 + q1;
                packed[j >> 1] |= ((uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8))
                                  << (16 * (j & 1));
            }
            const uint2 pv = make_uint2(packed[0], packed[1]);
            reinterpret_cast<uint2*>(xq + (size_t)t * H)[c] = pv;
            if (dbg_xq) reinterpret_cast<uint2*>(dbg_xq + (size_t)t * H)[c] = pv;
            if (tplanes) {
                // 8 codes -> one 32-bit word of each plane (word c % 4 of block c / 4)
                uint32_t d[3] = {0u, 0u, 0u};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t tc = lut[(packed[e >> 2] >> (8 * (e & 3))) & 0xffu];
                    d[0] |= (tc & 0xFu) << (4 * e);
                    d[1] |= ((tc >> 4) & 0xFu) << (4 * e);
                    d[2] |= (tc >> 8) << (4 * e);
                }
                uint32_t* dst = reinterpret_cast<uint32_t*>(tplanes + ((size_t)t * (H / 32) + (c >> 2)) * 48) + (c & 3);
                dst[0] = d[0];
                dst[4] = d[1];
                dst[8] = d[2];
            }
        }
        bsum += __shfl_xor_sync(0xffffffffu, bsum, 1);
        bsum += __shfl_xor_sync(0xffffffffu, bsum, 2);
        if (c < nchunk && (c & 3) == 0) xinit[(size_t)t * (H / 32) + (c >> 2)] = -12 * bsum;
    }
}

// ---- plan ----------------------------------------------------------------------------
// Work split per expert: experts with at least tc_min rows go to the
// tensor-core GEMM (tiles of tc_tile1 / tc_tile2 token rows x tc_wtile1 /
// tc_wtile2 weight rows of W1 / W2, the tiles of the forms and configurations
// those GEMMs are launched with; a ragged last weight block counts as a tile),
// the others to the streaming GEMM (units of kGemvTileRows weight rows
// x `group` tokens, the group size the streaming GEMM is launched with).  Forms the exclusive scans over experts of the streaming
// units of W1/W2, of the tensor-core tiles of W1/W2 and of the digit-plane rows
// (each tensor-core expert's rows padded to a multiple of 16, so that every
// tile starts on a 16-row boundary of the plane buffers), of the rows of
// streaming experts (their compact streaming rows), and expert_tc[e] = 1 for
// tensor-core experts.  Run by one warp; lane l owns a contiguous slice of
// experts.  The tables go to ps (shared memory) and, with global_out, to the
// global tables the GEMM launches index.
struct PlanShared {
    int32_t plane_off[kMaxExperts];
    int32_t stream_off[kMaxExperts];
    uint8_t tc[kMaxExperts];
    int32_t units1;   // streaming units of W1 (0: no streaming rows)
};

// The per-row slot table (plane_row) the planner writes for every sorted row:
// a value >= 0 is the digit-plane row of a tensor-core row; a negative value v
// marks a streaming row whose compact streaming row is ~v (its fp64
// accumulators, h codes and block terms live at that row of buffers sized for
// the streaming rows only); kNoRow marks a row that failed the planner's
// bounds check (its kernels skip it).
constexpr int32_t kNoRow = INT32_MIN;

static __device__ void plan_warp(const int32_t* __restrict__ offsets, int E, int P, int n1, int n2, int tc_min,
                                 int tc_tile1, int tc_tile2, int tc_wtile1, int tc_wtile2, int group,
                                 int32_t* __restrict__ unit_off1, int32_t* __restrict__ unit_off2,
                                 int32_t* __restrict__ tile_off1, int32_t* __restrict__ tile_off2,
                                 int32_t* __restrict__ plane_off, int32_t* __restrict__ stream_off,
                                 int32_t* __restrict__ expert_tc, int32_t* flag, bool global_out, PlanShared& ps) {
    constexpr int NS = 6;
    const int lane = threadIdx.x & 31;
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    // offsets must run from 0 up to at most P without decreasing; otherwise no
    // expert gets any work (and FLAG_BOUNDS is raised)
    bool bad = (lane == 0 && offsets[0] != 0) || (lane == 31 && offsets[E] > P);
    for (int e = e0; e < e1; ++e) bad |= offsets[e + 1] < offsets[e];
    const bool any_bad = __any_sync(0xffffffffu, bad);
    if (any_bad && lane == 0 && global_out) raise_flag(flag, FLAG_BOUNDS);
    auto counts = [&](int e, int (&c)[NS]) {
        const int m = any_bad ? 0 : offsets[e + 1] - offsets[e];
        const bool tc = m >= tc_min;
        const int g = tc ? 0 : (m + group - 1) / group;
        const int nb1 = tc ? (m + tc_tile1 - 1) / tc_tile1 : 0;
        const int nb2 = tc ? (m + tc_tile2 - 1) / tc_tile2 : 0;
        c[0] = g * (n1 / kGemvTileRows);
        c[1] = g * (n2 / kGemvTileRows);
        c[2] = nb1 * ((n1 + tc_wtile1 - 1) / tc_wtile1);
        c[3] = nb2 * ((n2 + tc_wtile2 - 1) / tc_wtile2);
        c[4] = tc ? (m + 15) & ~15 : 0;
        c[5] = tc ? 0 : m;
    };
    int s[NS] = {};
    for (int e = e0; e < e1; ++e) {
        int c[NS];
        counts(e, c);
        for (int j = 0; j < NS; ++j) s[j] += c[j];
    }
    int x[NS];
    for (int j = 0; j < NS; ++j) x[j] = s[j];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int j = 0; j < NS; ++j) {
            const int y = __shfl_up_sync(0xffffffffu, x[j], o);
            if (lane >= o) x[j] += y;
        }
    }
    int r[NS];
    for (int j = 0; j < NS; ++j) r[j] = x[j] - s[j];  // exclusive prefix
    int32_t* outs[NS] = {unit_off1, unit_off2, tile_off1, tile_off2, plane_off, stream_off};
    for (int e = e0; e < e1; ++e) {
        int c[NS];
        counts(e, c);
        const bool tc = !any_bad && (offsets[e + 1] - offsets[e]) >= tc_min;
        ps.plane_off[e] = r[4];
        ps.stream_off[e] = r[5];
        ps.tc[e] = tc ? 1 : 0;
        if (global_out) {
            for (int j = 0; j < NS; ++j) outs[j][e] = r[j];
            expert_tc[e] = tc ? 1 : 0;
        }
        for (int j = 0; j < NS; ++j) r[j] += c[j];
    }
    if (lane == 31) {
        ps.units1 = x[0];
        if (global_out)
            for (int j = 0; j < NS; ++j) outs[j][E] = x[j];
    }
}

}  // namespace moe
