// Streaming grouped GEMM for the decode regime (few tokens per expert).
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) drives its decode expert
// GEMMs from packed FP4 weights and INT8 activations with integer
// dot-product instructions, and names memory bandwidth and low M as the
// limits.  On B200 the same regime is HBM-bound: every touched expert's FP4
// weights are read exactly once, in coalesced 16-byte pieces.
//
// Work: for every expert e with M_e > 0, units (tile of kGemvTileRows = 64
// weight rows, group of up to kGroup tokens); each unit is K/128 items of 4
// scale blocks.  The
// flat item range is split evenly over all warps of the grid (stream-K), so
// the load is balanced to within one item whatever the expert counts are.
//
// Every warp runs its own kStages-deep ring in shared memory: the cp.async
// copies of item i + 1 -- the weights (every lane copies its own 16-byte code
// slices, a warp-wide 512-byte coalesced access per block), the group's
// activation bytes and block terms -- are in flight while item i is computed.
//
// Lane l of a warp owns weight rows 64*tile + l and 64*tile + 32 + l (two
// independent dot-product chains per lane, which share the activation loads)
// and their full dot products with the group's token rows:
//   * a 16-byte code slice gives the lane one 32-element block (one scale) of
//     one row; the warp's 32 slices of a block are one contiguous 512-byte
//     piece of the packed chunk, the two rows' pieces are adjacent (layout in
//     pack.cu);
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

// Tuning (measured on B200, decode T=8 and T=64): two adjacent 32-row tiles
// per warp (a lane owns two rows) with a 2-deep ring, 20 warps per SM (shared
// memory bound), beat one tile per warp at 32 warps per SM by 5-8% (decode_T8:
// 3.93 -> 4.19 TB/s): the second row gives every lane a second independent
// chain and halves the activation loads and the per-item bookkeeping per
// weight.  Four tiles per warp (11 warps per SM), a 3-deep ring (14 warps),
// one-tile variants with more or fewer registers, and TMA bulk copies in place
// of the per-lane 16-byte copies were all slower.  The kernel is bound by
// integer issue (the nibble decode), at about 0.65 of the measured copy
// bandwidth.  With the equal split the warps of a launch finish over a wide
// window (decode T = 8, W1: 32-81 us after the wait, in the order of their
// issue priority on the SM's schedulers); dynamic chunks from an atomic
// counter, a split weighted by priority, and an L2 prefetch a few items ahead
// all measured slower than the equal split.
// One warp per CTA, 32 CTAs per SM: every warp runs its own pipeline anyway,
// and single-warp CTAs measured ~10% faster than 8-warp CTAs at the same 32
// warps per SM (decode_T8: 3.58 -> 3.96 TB/s; 4 warps/CTA: 3.70).
constexpr int kGemvWarps = 1;
constexpr int kStages = 2;                   // shared-memory ring depth per warp
constexpr int kMinBlocks = 18;               // register budget: CTAs per SM (shared memory allows 20)
constexpr int TP = kGemvTileRows / 32;       // 32-row tiles per unit: a lane owns TP rows
static_assert(TP == 1 || TP == 2 || TP == 4, "a lane's scale words are one 4-, 8- or 16-byte copy");
constexpr int kScaleBytes = 32 * 4 * TP;     // the lanes' scale words (TP per lane)
constexpr int kGroupBytes = kScaleBytes + 4 * TP * 512;  // + 4 blocks x TP tiles x 512 B codes
constexpr int kChunkBytes = 8704;  // packed chunk: 4 scale blocks of 128 rows (see pack.cu)

// One ring slot: one K group (4 blocks of 32 elements) of one unit's TP
// 32-row tiles -- the lanes' scale words, then per block the TP tiles' 512-byte
// code slices -- plus the group's activation bytes and block terms.
// G = token rows per unit (2 or 4): the slot holds G activation rows, so a
// smaller group leaves room for more warps per SM.
template <int G>
struct alignas(16) Slot {
    uint8_t w[kGroupBytes];
    int8_t x[G][128];
    int32_t init[G][4];
};
template <int G>
constexpr int slot_bytes() { return (int)sizeof(Slot<G>); }
template <int G>
constexpr int smem_bytes() { return kGemvWarps * kStages * slot_bytes<G>(); }

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
constexpr uint32_t kPos0 = 0x0F0E0D0Cu, kPos1 = 0x18141210u;  // 12 + {0,1,2,3,4,6,8,12}
constexpr uint32_t kNeg0 = 0x090A0B0Cu, kNeg1 = 0x00040608u;  // 12 - {0,1,2,3,4,6,8,12}

// The four table words, held in registers for the whole kernel.  They are
// derived from a kernel argument that is always zero, so that the compiler
// keeps them in registers instead of re-materialising the immediates before
// every byte permute.
struct Tables {
    uint32_t p0, p1, n0, n1;
    __device__ __forceinline__ explicit Tables(uint32_t zero)
        : p0(kPos0 ^ zero), p1(kPos1 ^ zero), n0(kNeg0 ^ zero), n1(kNeg1 ^ zero) {}
};

__device__ __forceinline__ void decode8(const Tables& t, uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t wf = w ^ 0x88888888u;
    lo = prmt(t.p0, t.p1, w) | prmt(t.n0, t.n1, wf);
    hi = prmt(t.p0, t.p1, w >> 16) | prmt(t.n0, t.n1, wf >> 16);
}

// High word of the double 2^(S-128) for scale byte bb of the packed word sw:
// one byte permute and one multiply-add ((S + 895) << 20).
__device__ __forceinline__ double block_scale(uint32_t sw, int bb) {
    const uint32_t S = __byte_perm(sw, 0u, 0x4440u + (uint32_t)bb);
    return __hiloint2double((int)(S * 1048576u + 895u * 1048576u), 0);
}

__device__ __forceinline__ void cp_async16(uint32_t smem, const void* gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

struct GemvArgs {
    const uint8_t* w;          // matrix region of the packed buffer
    size_t expert_bytes;
    int K;                     // inputs per weight row
    int N;                     // weight rows per expert (= output columns)
    const int8_t* act;         // activation codes, rows of K bytes
    const int32_t* act_init;   // rows of K/32 block terms
    const int32_t* perm;       // sorted row -> pair id
    int k_div;                 // >0: activation row = perm[i] / k_div (sorted row i); 0: = the streaming row
    const int32_t* offsets;    // [E+1]
    const int32_t* unit_off;   // [E+1] exclusive scan of units per expert
    const int32_t* stream_off; // [E+1] first compact streaming row of each expert
    int E;
    double* out;               // [streaming rows, N] fp64 accumulators, zeroed
    const int32_t* flag;       // device error word: a layout mismatch stops the kernel
    int gate_up_half;          // > 0 (= I) for W1: device rows interleave gate and up rows
    int P;                     // pairs (rows of the sorted tables)
    int pre_wait;              // 1: the tables were written at least two launches back (see k_gemv)
    uint32_t zero;             // always 0 (see Tables)
};

// Canonical row (output column) of a device row (see the layout in pack.cu).
__device__ __forceinline__ int canonical_row(int d, int gate_up_half) {
    if (gate_up_half <= 0) return d;
    const int tau = d >> 5, r = d & 31;
    return (r < 16) ? tau * 16 + r : gate_up_half + tau * 16 + (r - 16);
}

// A unit: expert, tile, first sorted row, its compact streaming row, number of rows.
struct Unit {
    int id, e, tile, i0, o0, mc;
};

template <int G>
__device__ __forceinline__ Unit unit_at(const GemvArgs& a, int unit) {
    // (callers stay inside the launch's units; a unit past them would address
    // memory outside the tables and weights, so it is flagged and clamped)
    const int units = __ldg(a.unit_off + a.E);
    if (unit >= units) {
        raise_flag(const_cast<int32_t*>(a.flag), FLAG_BOUNDS);
        unit = units - 1;
    }
    int lo = 0, hi = a.E;  // last e with unit_off[e] <= unit
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(a.unit_off + mid) <= unit) lo = mid; else hi = mid;
    }
    Unit u;
    u.id = unit;
    u.e = lo;
    const int r0 = __ldg(a.offsets + lo), r1 = __ldg(a.offsets + lo + 1);
    const int ngroups = (r1 - r0 + G - 1) / G;
    const int local = unit - __ldg(a.unit_off + lo);
    u.tile = local / ngroups;
    u.i0 = r0 + (local % ngroups) * G;
    u.o0 = __ldg(a.stream_off + lo) + (u.i0 - r0);
    u.mc = min(G, r1 - u.i0);
    return u;
}

// Activation row of row m of unit u: the token (W1) or the streaming row (W2).
__device__ __forceinline__ int act_row(const GemvArgs& a, const Unit& u, int m) {
    return a.k_div ? checked_index(__ldg(a.perm + u.i0 + m), a.P, const_cast<int32_t*>(a.flag)) / a.k_div
                   : u.o0 + m;
}

// Integer dot product of one 32-element block (8 decoded words) with one
// token's 32 activation bytes, started from the block term.
__device__ __forceinline__ int block_dot(const uint32_t (&v)[8], const uint4& x0, const uint4& x1,
                                         int init) {
    int d0 = init, d1 = 0;
    d0 = __dp4a((int)v[0], (int)x0.x, d0);
    d1 = __dp4a((int)v[1], (int)x0.y, d1);
    d0 = __dp4a((int)v[2], (int)x0.z, d0);
    d1 = __dp4a((int)v[3], (int)x0.w, d1);
    d0 = __dp4a((int)v[4], (int)x1.x, d0);
    d1 = __dp4a((int)v[5], (int)x1.y, d1);
    d0 = __dp4a((int)v[6], (int)x1.z, d0);
    d1 = __dp4a((int)v[7], (int)x1.w, d1);
    return d0 + d1;
}

// Single-token variant: the positive- and negative-table bytes of each word
// feed two dot products instead of being merged first (the merge moves from
// the ALU pipe to dp4a), worthwhile when one token carries the whole decode.
__device__ __forceinline__ int block_dot_split(const Tables& t, const uint4& c, const uint4& x0,
                                               const uint4& x1, int init) {
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    int d0 = init, d1 = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t w = cw[j], wf = w ^ 0x88888888u;
        d0 = __dp4a((int)prmt(t.p0, t.p1, w), (int)xw[2 * j], d0);
        d1 = __dp4a((int)prmt(t.n0, t.n1, wf), (int)xw[2 * j], d1);
        d0 = __dp4a((int)prmt(t.p0, t.p1, w >> 16), (int)xw[2 * j + 1], d0);
        d1 = __dp4a((int)prmt(t.n0, t.n1, wf >> 16), (int)xw[2 * j + 1], d1);
    }
    return d0 + d1;
}

// Warps per SM are bounded by each scheduler's 16 K registers (5 warps of up to
// 96 registers, 6 of up to 80) and by shared memory (one-warp CTAs with two
// slots: 21 for G = 4, 22 for G = 2).  G = 4 keeps 86 registers (5 warps per
// scheduler, 20 per SM); G = 2 is held to at most 80 so that its smaller slots
// can fill 22 warps.
template <int G>
__global__ void __launch_bounds__(kGemvWarps * 32, G == 2 ? 25 : kMinBlocks) k_gemv(GemvArgs a) {
    constexpr int kGroup = G;
    using Slot = moe::Slot<G>;
    constexpr int kSlotBytes = slot_bytes<G>();
    // pre_wait: the launch in front of this one (the h quant, in front of W2)
    // writes only the activations, and the unit tables and the error word's
    // FLAG_LAYOUT bit come from launches before it, which had completed when
    // that launch passed its own wait.  So the weights of the warp's first item
    // go into the ring while the launch in front still runs, and the
    // activations are copied after the wait.  (Also prefetching the next items'
    // weights into L2 there measured slower: it delayed the h quant.)
    if (!a.pre_wait) pdl_begin();
    extern __shared__ __align__(16) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // packed weights built for other dims may be smaller than the offsets used here
    if (*(volatile const int32_t*)a.flag & FLAG_LAYOUT) return;
    const Tables tb(a.zero);
    Slot* ring = reinterpret_cast<Slot*>(smem) + warp * kStages;
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    const long long gw = (long long)blockIdx.x * kGemvWarps + warp;
    const long long nw = (long long)gridDim.x * kGemvWarps;
    const int KG = a.K / 128;
    const long long W = (long long)__ldg(a.unit_off + a.E) * KG;
    const int it0 = (int)(W * gw / nw), it1 = (int)(W * (gw + 1) / nw);
    if (it0 >= it1) return;

    // per-lane byte offsets inside a slot: own scale word, own code slices, the
    // 16-byte activation chunk (token lane/8, chunk lane%8) and block terms
    // (token lane%4) this lane copies.  In the packed chunk of 8704 bytes the
    // lane's scale word of tile t is at lane*16 + t*4 and its code slice of
    // block j at 512 + j*2048 + t*512 + lane*16.
    const uint32_t o_sc = lane * 4 * TP, o_code = kScaleBytes + lane * 16;
    const uint32_t o_x = (uint32_t)offsetof(Slot, x) + (lane >> 3) * 128 + (lane & 7) * 16;
    const uint32_t o_init = (uint32_t)offsetof(Slot, init) + (lane & (kGroup - 1)) * 16;

    // ---- fetch side: cp.async copies of one item into its slot ----
    int f_left = it1 - it0;
    int f_kg = it0 % KG, f_slot = 0;
    Unit fu = unit_at<G>(a, it0 / KG);
    const uint8_t* f_w = nullptr;  // this lane's sources for the current item
    const int8_t* f_x = nullptr;
    const int32_t* f_i = nullptr;
    uint32_t g_sc = 0, g_code = 0;  // this lane's offsets inside a packed chunk (tile dependent)
    auto start_unit = [&](int kg) {
        const int rb = (fu.tile * TP) >> 2, t = (fu.tile * TP) & 3;
        g_sc = lane * 16 + t * 4;
        g_code = 512 + t * 512 + lane * 16;
        f_w = a.w + (size_t)fu.e * a.expert_bytes + ((size_t)rb * KG + kg) * kChunkBytes;
        f_x = a.act + (size_t)act_row(a, fu, min(lane >> 3, fu.mc - 1)) * a.K + kg * 128 + (lane & 7) * 16;
        f_i = a.act_init + (size_t)act_row(a, fu, min(lane & (kGroup - 1), fu.mc - 1)) * (a.K / 32) +
              kg * 4;
    };
    start_unit(f_kg);
    auto issue_w = [&]() {  // the item's weights
        const uint32_t sb = ring_s + f_slot * kSlotBytes;
        if (TP == 4) cp_async16(sb + o_sc, f_w + g_sc);
        else if (TP == 2) cp_async8(sb + o_sc, f_w + g_sc);
        else cp_async4(sb + o_sc, f_w + g_sc);
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
#pragma unroll
            for (int u = 0; u < TP; ++u)
                cp_async16(sb + o_code + (bb * TP + u) * 512, f_w + g_code + bb * 2048 + u * 512);
    };
    auto issue_x = [&]() {  // the item's activation bytes and block terms
        const uint32_t sb = ring_s + f_slot * kSlotBytes;
        if ((lane >> 3) < fu.mc) cp_async16(sb + o_x, f_x);
        if (lane < fu.mc) cp_async16(sb + o_init, f_i);
    };
    auto advance = [&]() {  // to the next item of the warp's range
        --f_left;
        f_slot = (f_slot + 1 == kStages) ? 0 : f_slot + 1;
        if (++f_kg == KG) {
            if (f_left > 0) {
                f_kg = 0;
                fu = unit_at<G>(a, fu.id + 1);
                start_unit(0);
            }
        } else {
            f_w += kChunkBytes;
            f_x += 128;
            f_i += 4;
        }
    };
    auto issue = [&]() {
        issue_w();
        issue_x();
        cp_async_commit();
        advance();
    };

    static_assert(kStages == 2, "the prologue fills one slot");
    if (a.pre_wait) {  // (f_left > 0 here)
        issue_w();
        cp_async_commit();
        pdl_begin();
        issue_x();
        cp_async_commit();
        advance();
    } else {
        issue();
    }

    // ---- compute side ----
    Unit cu = unit_at<G>(a, it0 / KG);
    int c_kg = it0 % KG, c_slot = 0;
    double acc[TP][kGroup];
#pragma unroll
    for (int u = 0; u < TP; ++u)
#pragma unroll
        for (int m = 0; m < kGroup; ++m) acc[u][m] = 0.0;
    for (int it = it0; it < it1; ++it) {
        if (f_left > 0) issue();
        else cp_async_commit();
        cp_async_wait<kStages - 1>();  // item `it` has landed (this lane's copies) ...
        __syncwarp();                  // ... and every other lane's
        const Slot& sl = ring[c_slot];
        uint32_t sw[TP];
#pragma unroll
        for (int u = 0; u < TP; ++u) sw[u] = *reinterpret_cast<const uint32_t*>(sl.w + o_sc + 4 * u);
        if (cu.mc == 1) {
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const uint4 x0 = *reinterpret_cast<const uint4*>(&sl.x[0][bb * 32]);
                const uint4 x1 = *reinterpret_cast<const uint4*>(&sl.x[0][bb * 32 + 16]);
                const int ini = sl.init[0][bb];
#pragma unroll
                for (int u = 0; u < TP; ++u) {
                    const uint4 c = *reinterpret_cast<const uint4*>(sl.w + o_code + (bb * TP + u) * 512);
                    const int d = block_dot_split(tb, c, x0, x1, ini);
                    acc[u][0] = __fma_rn((double)d, block_scale(sw[u], bb), acc[u][0]);
                }
            }
        } else {
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                uint32_t v[TP][8];
                double sc[TP];
#pragma unroll
                for (int u = 0; u < TP; ++u) {
                    const uint4 c = *reinterpret_cast<const uint4*>(sl.w + o_code + (bb * TP + u) * 512);
                    decode8(tb, c.x, v[u][0], v[u][1]);
                    decode8(tb, c.y, v[u][2], v[u][3]);
                    decode8(tb, c.z, v[u][4], v[u][5]);
                    decode8(tb, c.w, v[u][6], v[u][7]);
                    sc[u] = block_scale(sw[u], bb);
                }
#pragma unroll
                for (int m = 0; m < kGroup; ++m) {
                    if (m < cu.mc) {
                        const uint4 x0 = *reinterpret_cast<const uint4*>(&sl.x[m][bb * 32]);
                        const uint4 x1 = *reinterpret_cast<const uint4*>(&sl.x[m][bb * 32 + 16]);
                        const int ini = sl.init[m][bb];
#pragma unroll
                        for (int u = 0; u < TP; ++u)
                            acc[u][m] = __fma_rn((double)block_dot(v[u], x0, x1, ini), sc[u], acc[u][m]);
                    }
                }
            }
        }
        __syncwarp();  // every lane is done with the slot before it is refilled
        c_slot = (c_slot + 1 == kStages) ? 0 : c_slot + 1;
        if (++c_kg == KG || it + 1 == it1) {
#pragma unroll
            for (int u = 0; u < TP; ++u) {
                const int n = canonical_row((cu.tile * TP + u) * 32 + lane, a.gate_up_half);
#pragma unroll
                for (int m = 0; m < kGroup; ++m) {
                    if (m < cu.mc) atomicAdd(a.out + (size_t)(cu.o0 + m) * a.N + n, acc[u][m]);
                    acc[u][m] = 0.0;
                }
            }
            if (c_kg == KG && it + 1 < it1) {
                c_kg = 0;
                cu = unit_at<G>(a, cu.id + 1);
            }
        }
    }
    cp_async_wait<0>();
}

template <int G>
static int gemv_grid() {
    static PerContext cache;
    return cache.get([] {
        int dev = 0, sms = 0, per_sm = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaFuncSetAttribute(k_gemv<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes<G>()) !=
                cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv<G>, kGemvWarps * 32, smem_bytes<G>()) !=
                cudaSuccess)
            return -1;
        return sms * (per_sm > 0 ? per_sm : 1);
    });
}

cudaError_t launch_gemv(const uint8_t* w, size_t expert_bytes, int K, int N, const int8_t* act,
                        const int32_t* act_init, const int32_t* perm, int k_div,
                        const int32_t* offsets, const int32_t* unit_off, const int32_t* stream_off, int E,
                        double* out, const int32_t* flag, int gate_up_half, int P, int group, bool pre_wait,
                        cudaStream_t st) {
    GemvArgs a{w, expert_bytes, K, N, act, act_init, perm, k_div, offsets, unit_off, stream_off, E, out, flag,
               gate_up_half, P, pre_wait ? 1 : 0, 0u};
    const int grid = group == 2 ? gemv_grid<2>() : gemv_grid<4>();
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    const cudaError_t e =
        group == 2 ? launch_pdl(k_gemv<2>, dim3(grid), dim3(kGemvWarps * 32), smem_bytes<2>(), st, a)
                   : launch_pdl(k_gemv<4>, dim3(grid), dim3(kGemvWarps * 32), smem_bytes<4>(), st, a);
    count_launches(1);
    return e;
}

}  // namespace moe
