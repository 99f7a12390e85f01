// FP8 block-quantised dense projection on the tensor cores.
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) runs the model's dense
// projections in FP8; "DeepSeek V4 Flash on 8x R9600D" (model facts) names the
// format "FP8 block quantization".  The computation (readings in the header):
//   xq, sx  per token and 128-input block of x: sx = the smallest power of two
//           2^e with max|x| <= 448 * 2^e (UE8M0 byte e + 127), xq = E4M3 codes
//           of x / 2^e, round to nearest even;
//   y[t, n] = bf16( sum_k xq[t,k] 2^(sx[t,k/128]-127) * wq[n,k] 2^(sw[n/128,k/128]-127) )
// with E4M3 weight codes wq [N, K] and one UE8M0 scale per 128 x 128 weight
// block.  On B200 the contraction is tcgen05.mma kind::mxf8f6f4 with block
// scaling (E4M3 x E4M3, one UE8M0 factor per 32 inputs: each 128-input block
// scale is repeated over its four 32-input blocks), fp32 accumulation in TMEM.
//
// Layouts (both operands K-major, no swizzle, 8-row x 16-byte core matrices):
//   weights: 128-row x 128-input chunks of 16,896 bytes, chunk (rb, g) of the
//     N/128 x K/128 grid at (rb * K/128 + g) * 16896 after a 256-byte header:
//     512 scale bytes in the tensor cores' 128 x 4 scale-factor atom (byte
//     l*16 + t*4 + j for row t*32 + l, 32-input block j; all equal here), then
//     for each 16-input column c the 128 rows' 16-byte pieces (2 KB, 8-row
//     groups of 128 bytes).
//   activations: for token tile nb (128 tokens) and 128-input stage g, 16 KB
//     of codes at (nb * K/128 + g) * 16384, ordered by 8-token group: group r8
//     holds its 8 16-input columns' core matrices (128 bytes each) in 1 KB, so
//     the first n tokens of a tile are one contiguous n * 128 bytes; and 512
//     scale bytes in the atom at (nb * K/128 + g) * 512 of a second region.
// One stage of the GEMM is one bulk copy each of the weight chunk, the tile's
// token rows (rounded up to 16) and the scale block; four MMAs (K = 32 each)
// consume it.
//
// Kernel: one persistent CTA per SM with the roles of the FP4 expert GEMM
// (two producer / MMA-issuer pipes on alternate tiles, three 128-column TMEM
// accumulators, 16 epilogue warps), tiles of 128 weight rows x 128 tokens,
// token-tile-major so that consecutive tiles share the activations in L2.
// The epilogue writes bf16 y.  Every wait is bounded and raises
// MOE_FLAG_TIMEOUT.
// Decode sizes (T <= kFp8SplitMaxT: one token tile, N/128 tiles for 148 SMs):
// the K range of every tile is split over S CTAs (S <= 8, about SMs / tiles),
// each writes its fp32 partial sums to the workspace, and k_fp8_reduce adds
// the S partials in a fixed order and rounds to bf16 -- deterministic, and the
// weight stream is spread over S times as many SMs.
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "moe_common.cuh"
#include "tcgen05.cuh"

namespace moe {

constexpr int F8_BM = 128, F8_BN = 128;
constexpr int F8_PIPES = 2, F8_STAGES = 3, F8_ACC = 3;
constexpr int F8_A_BYTES = kFp8ChunkBytes;            // 512 scale bytes + 128 x 128 codes
constexpr int F8_B_BYTES = 128 * 128;                 // 128 tokens x 128 inputs
constexpr int F8_SF_BYTES = 512;
constexpr int F8_STAGE_BYTES = F8_A_BYTES + F8_B_BYTES + F8_SF_BYTES;
constexpr int F8_EPI_WARPS = 16;
constexpr int F8_EPI_WARP0 = 2 * F8_PIPES;
constexpr int F8_THREADS = 32 * (F8_EPI_WARP0 + F8_EPI_WARPS);
constexpr int F8_TMEM_COLS = 512;
// TMEM columns: accumulators at b * 128; per pipe r and stage s the A scale
// factors at F8_SF_COL + 8 (F8_STAGES r + s) and the B scale factors 4 after.
constexpr int F8_SF_COL = F8_ACC * F8_BN;
static_assert(F8_SF_COL + F8_PIPES * F8_STAGES * 8 <= F8_TMEM_COLS, "TMEM columns");

struct F8Shared {
    uint8_t stage[F8_PIPES][F8_STAGES][F8_STAGE_BYTES];
    uint64_t full[F8_PIPES][F8_STAGES], empty[F8_PIPES][F8_STAGES], acc_full[F8_ACC], acc_empty[F8_ACC];
    uint64_t drain[F8_PIPES];
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(F8Shared) <= 227 * 1024, "shared memory per CTA");

struct F8Args {
    const uint8_t* w;          // first chunk (after the header)
    const uint8_t* xb;         // activation code blocks
    const uint8_t* xs;         // activation scale blocks
    int T, N, K;
    __nv_bfloat16* y;          // [T, N]
    int32_t* flag;
    uint64_t wait_ns;
    int splits;                // S > 1: K split S ways, fp32 partials to `part`
    float* part;               // [S][T][N]
};

// kind::mxf8f6f4 instruction descriptor: E4M3 x E4M3, UE8M0 scales, fp32
// accumulate, K-major operands, M = 128; the scale-factor ids pick the 32-input
// block of the stage.
__device__ __forceinline__ uint32_t f8_idesc(int n, int sf_id) {
    uint32_t d = 0;
    d |= (uint32_t)(sf_id & 3) << 4;      // B scale factor id
    // A and B formats: E4M3 = 0 (bits 7-9, 10-12)
    d |= (uint32_t)(n >> 3) << 17;        // N / 8
    d |= 1u << 23;                        // scale format UE8M0
    d |= (uint32_t)(F8_BM >> 4) << 24;    // M / 16
    d |= (uint32_t)(sf_id & 3) << 29;     // A scale factor id
    return d;
}

__device__ __forceinline__ void tc_mma_mxf8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

__global__ void __launch_bounds__(F8_THREADS, 1) k_fp8_gemm(F8Args a) {
    pdl_begin();
    // weights packed for other dims: their chunks are not where this call looks
    if (*(volatile int32_t*)a.flag & FLAG_LAYOUT) return;
    extern __shared__ __align__(1024) uint8_t f8_smem_raw[];
    F8Shared& sh = *reinterpret_cast<F8Shared*>(f8_smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KG = a.K / 128, RB = a.N / F8_BM, NB = (a.T + F8_BN - 1) / F8_BN, S = a.splits;
    const int total = RB * NB * S;
    if (total == 0) return;
    const int ntiles = ((int)blockIdx.x < total) ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    // work item j of this CTA: tile (rb, nb) and its K range [g0, g1)
    auto tile = [&](int j, int& rb, int& nb, int& g0, int& g1, int& s) {
        const int t = (int)blockIdx.x + j * (int)gridDim.x;
        const int tt = t / S;
        s = t % S;
        nb = tt / RB;
        rb = tt % RB;
        g0 = s * KG / S;
        g1 = (s + 1) * KG / S;
    };

    if (threadIdx.x == 0) {
        for (int r = 0; r < F8_PIPES; ++r)
            for (int s = 0; s < F8_STAGES; ++s) {
                mbar_init(smem_u32(&sh.full[r][s]), 1);
                mbar_init(smem_u32(&sh.empty[r][s]), 1);
            }
        for (int b = 0; b < F8_ACC; ++b) {
            mbar_init(smem_u32(&sh.acc_full[b]), 1);
            mbar_init(smem_u32(&sh.acc_empty[b]), F8_EPI_WARPS);
        }
        for (int r = 0; r < F8_PIPES; ++r) mbar_init(smem_u32(&sh.drain[r]), 1);
        sh.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem_base)),
                     "r"(F8_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int32_t* abort = &sh.abort;
    auto give_up = [&]() {
        *abort = 1;
        raise_flag(a.flag, FLAG_TIMEOUT);
    };
    auto wait = [&](uint32_t bar, uint32_t parity) { return mbar_wait_for<false>(bar, parity, a.wait_ns, abort); };
    auto final_wait = [&](uint32_t bar, uint32_t parity) {
        if (!mbar_wait_for<false>(bar, parity, a.wait_ns, nullptr)) raise_flag(a.flag, FLAG_TIMEOUT);
    };

    if (warp < F8_PIPES) {
        // ---------------- producer of pipe r ----------------
        const int r = warp;
        int stage = 0;
        uint32_t phase = 0;
        bool filled[F8_STAGES] = {};
        uint32_t fill_parity[F8_STAGES] = {};
        for (int j = r; j < ntiles && !*abort; j += F8_PIPES) {
            int rb, nb, g0, g1, sp;
            tile(j, rb, nb, g0, g1, sp);
            const uint8_t* wsrc = a.w + (size_t)rb * KG * F8_A_BYTES;
            const uint8_t* bsrc = a.xb + (size_t)nb * KG * F8_B_BYTES;
            const uint8_t* ssrc = a.xs + (size_t)nb * KG * F8_SF_BYTES;
            const int n_mma = (min(F8_BN, a.T - nb * F8_BN) + 15) & ~15;
            const uint32_t bbytes = (uint32_t)n_mma * 128;   // the tile's token rows
            for (int g = g0; g < g1; ++g) {
                const uint32_t fb = smem_u32(&sh.full[r][stage]), eb = smem_u32(&sh.empty[r][stage]);
                if (!wait(eb, phase ^ 1u)) {
                    give_up();
                    break;
                }
                const uint32_t sbase = smem_u32(sh.stage[r][stage]);
                if (lane == 0) {
                    mbar_expect_tx(fb, F8_A_BYTES + bbytes + F8_SF_BYTES);
                    bulk_g2s(sbase, wsrc + (size_t)g * F8_A_BYTES, F8_A_BYTES, fb);
                    bulk_g2s(sbase + F8_A_BYTES, bsrc + (size_t)g * F8_B_BYTES, bbytes, fb);
                    bulk_g2s(sbase + F8_A_BYTES + F8_B_BYTES, ssrc + (size_t)g * F8_SF_BYTES, F8_SF_BYTES, fb);
                }
                __syncwarp();
                filled[stage] = true;
                fill_parity[stage] = phase;
                if (++stage == F8_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        for (int s = 0; s < F8_STAGES; ++s)
            if (filled[s] && lane == 0) final_wait(smem_u32(&sh.full[r][s]), fill_parity[s]);
        __syncwarp();
    } else if (warp < F8_EPI_WARP0) {
        // ---------------- MMA issuer of pipe r ----------------
        const int r = warp - F8_PIPES;
        int stage = 0;
        uint32_t phase = 0;
        for (int j = r; j < ntiles && !*abort; j += F8_PIPES) {
            int rb, nb, g0, g1, sp;
            tile(j, rb, nb, g0, g1, sp);
            const int n_valid = min(F8_BN, a.T - nb * F8_BN);
            const int n_mma = (n_valid + 15) & ~15;
            const int buf = j % F8_ACC;
            const uint32_t use = (uint32_t)(j / F8_ACC);
            if (!wait(smem_u32(&sh.acc_empty[buf]), (use & 1u) ^ 1u)) {
                give_up();
                break;
            }
            tc_fence_after();
            const uint32_t dcol = tmem + buf * F8_BN;
            bool ok = true;
            for (int g = g0; g < g1; ++g) {
                if (!wait(smem_u32(&sh.full[r][stage]), phase)) {
                    give_up();
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t sa = smem_u32(sh.stage[r][stage]);
                    const uint32_t sb = sa + F8_A_BYTES;
                    const uint32_t sfa = tmem + F8_SF_COL + 8 * (F8_STAGES * r + stage);
                    const uint32_t sfb = sfa + 4;
                    tc_cp_sf(sfa, make_sdesc(sa, 0, 128));
                    tc_cp_sf(sfb, make_sdesc(sb + F8_B_BYTES, 0, 128));
#pragma unroll
                    for (int mi = 0; mi < 4; ++mi) {
                        // inputs 32 mi .. 32 mi + 31: 16-byte columns 2 mi and 2 mi + 1
                        // (weights: columns 2 KB apart, 8-row groups 128 B apart;
                        // tokens: columns 128 B apart, 8-row groups 1 KB apart)
                        const uint64_t adesc = make_sdesc(sa + 512 + mi * 2 * 2048, 2048, 128);
                        const uint64_t bdesc = make_sdesc(sb + mi * 2 * 128, 128, 1024);
                        tc_mma_mxf8(dcol, adesc, bdesc, f8_idesc(n_mma, mi), sfa, sfb, (g > g0) || mi != 0);
                    }
                    tc_commit(smem_u32(&sh.empty[r][stage]));
                }
                __syncwarp();
                if (++stage == F8_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) tc_commit(smem_u32(&sh.acc_full[buf]));
            __syncwarp();
        }
        if (lane == 0) {
            tc_commit(smem_u32(&sh.drain[r]));
            final_wait(smem_u32(&sh.drain[r]), 0);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue ----------------
        // Warp (q, c): TMEM lane quadrant q (weight rows 32q..32q+31 of the
        // tile: output features) and 32-column chunk c (tokens).  Each thread
        // holds one output feature of 32 tokens and writes them as bf16.
        const int ew = warp - F8_EPI_WARP0;
        const int q = warp & 3;
        const int n0 = 32 * (ew >> 2);
        for (int j = 0; j < ntiles && !*abort; ++j) {
            int rb, nb, g0, g1, sp;
            tile(j, rb, nb, g0, g1, sp);
            const int n_valid = min(F8_BN, a.T - nb * F8_BN);
            const int buf = j % F8_ACC;
            const uint32_t use = (uint32_t)(j / F8_ACC);
            if (!wait(smem_u32(&sh.acc_full[buf]), use & 1u)) {
                give_up();
                break;
            }
            tc_fence_after();
            if (n0 < n_valid) {
                uint32_t v[32];
                tc_ld32(tmem + ((uint32_t)(q * 32) << 16) + buf * F8_BN + n0, v);
                const int n = rb * F8_BM + q * 32 + lane;
                if (S == 1) {
                    __nv_bfloat16* out = a.y + (size_t)(nb * F8_BN + n0) * a.N + n;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (n0 + c < n_valid) out[(size_t)c * a.N] = __float2bfloat16_rn(__uint_as_float(v[c]));
                } else {
                    float* out = a.part + ((size_t)sp * a.T + nb * F8_BN + n0) * a.N + n;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (n0 + c < n_valid) out[(size_t)c * a.N] = __uint_as_float(v[c]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.acc_empty[buf]));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(F8_TMEM_COLS)
                     : "memory");
}

// ---- activation quantisation into the GEMM's tiles ---------------------------
// One CTA (256 threads) per token; thread j takes 16 consecutive inputs of a
// 128-input block (8 threads per block, in one warp).  The block maximum is
// exact (bf16 inputs), the scale exponent the smallest e with a <= 448 * 2^e,
// the codes x / 2^e rounded to nearest even (cvt.rn.satfinite; the scaled
// values never exceed 448).
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(a), "f"(b));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(c), "f"(d));
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

// The first kernel of a call: thread 0 of CTA 0 also clears the call's error
// word, or sets FLAG_LAYOUT when the packed weights were built for other dims.
__global__ void __launch_bounds__(256)
    k_fp8_quant_act(const __nv_bfloat16* __restrict__ x, int T, int K, uint8_t* __restrict__ xb,
                    uint8_t* __restrict__ xs, uint8_t* __restrict__ dbg_q, uint8_t* __restrict__ dbg_s,
                    const uint8_t* __restrict__ packed, int N, int32_t* flag) {
    pdl_begin();
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        const Fp8Header* h = reinterpret_cast<const Fp8Header*>(packed);
        *flag = (h->magic == kFp8Magic && (int)h->N == N && (int)h->K == K) ? 0 : FLAG_LAYOUT;
    }
    const int t = blockIdx.x;
    const int KG = K / 128, nb = t / F8_BN, row = t % F8_BN;
    const int nchunk = K / 16;
    for (int c0 = 0; c0 < nchunk; c0 += blockDim.x) {
        const int ci = c0 + threadIdx.x;      // 16-input chunk; 8 per 128-input block
        const bool on = ci < nchunk;          // (nchunk % 8 == 0: a block's 8 lanes agree)
        float v[16];
        float amax = 0.0f;
        if (on) {
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * K + ci * 16);
            const uint4 p0 = __ldg(src), p1 = __ldg(src + 1);
            const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                v[2 * i] = __uint_as_float(w[i] << 16);
                v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
                amax = fmaxf(amax, fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1])));
            }
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        if (!on) continue;
        // smallest e with amax <= 448 * 2^e (exact comparisons of fp32 values)
        int e = -127;
        uint32_t sbyte = 0;
        if (amax > 0.0f) {
            int ea;
            frexpf(amax, &ea);                // amax in [2^(ea-1), 2^ea)
            e = max(-127, ea - 9);            // 448 * 2^(ea-10) < 2^(ea-1) <= amax, so e >= ea - 9
            while (amax > ldexpf(448.0f, e)) ++e;
            sbyte = (uint32_t)min(254, e + 127);
        }
        const float inv = amax > 0.0f ? ldexpf(1.0f, -e) : 0.0f;
        uint4 codes;
        codes.x = e4m3x4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
        codes.y = e4m3x4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
        codes.z = e4m3x4(v[8] * inv, v[9] * inv, v[10] * inv, v[11] * inv);
        codes.w = e4m3x4(v[12] * inv, v[13] * inv, v[14] * inv, v[15] * inv);
        const int g = ci / 8, col = ci % 8;
        uint8_t* dst = xb + ((size_t)nb * KG + g) * F8_B_BYTES + (row >> 3) * 1024 + col * 128 + (row & 7) * 16;
        *reinterpret_cast<uint4*>(dst) = codes;
        if (dbg_q) *reinterpret_cast<uint4*>(dbg_q + (size_t)t * K + ci * 16) = codes;
        if (col == 0) {
            uint8_t* sdst = xs + ((size_t)nb * KG + g) * F8_SF_BYTES + (row & 31) * 16 + (row >> 5) * 4;
            *reinterpret_cast<uint32_t*>(sdst) = sbyte * 0x01010101u;
            if (dbg_s) dbg_s[(size_t)t * KG + g] = (uint8_t)sbyte;
        }
    }
}

// ---- weight packing ------------------------------------------------------------
// Canonical wq [N, K] codes and ws [N/128, K/128] scale bytes <-> chunks.  A
// thread moves one 16-byte piece (or, for the first 32 threads of a chunk's
// pieces, 16 scale bytes).  fwd = false is the exact inverse (the scale of a
// chunk is read from its first byte).
__global__ void k_fp8_pack(const uint8_t* __restrict__ wq, const uint8_t* __restrict__ ws, uint8_t* __restrict__ chunks,
                           int N, int K, bool fwd, uint8_t* __restrict__ out_wq, uint8_t* __restrict__ out_ws,
                           int32_t* flag) {
    const int KG = K / 128;
    const size_t nchunks = (size_t)(N / 128) * KG;
    const size_t pieces = nchunks * (1024 + 32);  // 1024 code pieces + 32 scale pieces per chunk
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < pieces; i += (size_t)gridDim.x * blockDim.x) {
        const size_t ch = i / 1056;
        const int p = (int)(i % 1056);
        const int rb = (int)(ch / KG), g = (int)(ch % KG);
        uint8_t* base = chunks + ch * kFp8ChunkBytes;
        if (p < 32) {   // scale atom, 16 bytes per piece
            if (fwd) {
                const uint8_t sb = ws[(size_t)rb * KG + g];
                if (sb == 0xFF) raise_flag(flag, FLAG_BAD_SCALE);
                *reinterpret_cast<uint4*>(base + p * 16) = make_uint4(sb * 0x01010101u, sb * 0x01010101u,
                                                                     sb * 0x01010101u, sb * 0x01010101u);
            } else if (p == 0) {
                out_ws[(size_t)rb * KG + g] = base[0];
            }
            continue;
        }
        const int q = p - 32;                 // row r = q % 128, column c = q / 128
        const int r = q & 127, c = q >> 7;
        uint8_t* piece = base + 512 + c * 2048 + (r >> 3) * 128 + (r & 7) * 16;
        const size_t src = (size_t)(rb * 128 + r) * K + g * 128 + c * 16;
        if (fwd)
            *reinterpret_cast<uint4*>(piece) = *reinterpret_cast<const uint4*>(wq + src);
        else
            *reinterpret_cast<uint4*>(out_wq + src) = *reinterpret_cast<const uint4*>(piece);
    }
}

__global__ void k_fp8_header(uint8_t* packed, int N, int K) {
    Fp8Header* h = reinterpret_cast<Fp8Header*>(packed);
    h->magic = kFp8Magic;
    h->N = (uint32_t)N;
    h->K = (uint32_t)K;
    h->flag = 0;
}


size_t fp8_packed_bytes(int N, int K) { return kFp8HeaderBytes + (size_t)(N / 128) * (K / 128) * kFp8ChunkBytes; }

// Workspace: the error word (256 bytes), the activation tiles, then (calls of
// at most kFp8SplitMaxT tokens) the fp32 partial sums of the split K ranges.
static size_t fp8_act_bytes(int T, int K) {
    const size_t nb = (size_t)(T + F8_BN - 1) / F8_BN;
    return nb * (K / 128) * (F8_B_BYTES + F8_SF_BYTES);
}
static size_t fp8_part_offset(int T, int K) { return 256 + ((fp8_act_bytes(T, K) + 255) & ~(size_t)255); }

size_t fp8_workspace_bytes(int T, int N, int K) {
    // (a call with fewer tokens than T lays its partials out at a lower offset)
    const int tp = std::min(T, kFp8SplitMaxT);
    return fp8_part_offset(T, K) + (size_t)kFp8MaxSplits * tp * N * sizeof(float);
}

// y = bf16(sum over s of the partial sums, s = 0, 1, ... in order).
__global__ void __launch_bounds__(256)
    k_fp8_reduce(const float* __restrict__ part, int S, int T, int N, __nv_bfloat16* __restrict__ y,
                 const int32_t* flag) {
    pdl_begin();
    // weights packed for other dims: the GEMM wrote no partials and y stays untouched
    if (*(volatile const int32_t*)flag & FLAG_LAYOUT) return;
    const size_t tn = (size_t)T * N, n4 = tn / 4;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        float4 acc = reinterpret_cast<const float4*>(part)[i];
        for (int s = 1; s < S; ++s) {
            const float4 v = reinterpret_cast<const float4*>(part + (size_t)s * tn)[i];
            acc.x = __fadd_rn(acc.x, v.x);
            acc.y = __fadd_rn(acc.y, v.y);
            acc.z = __fadd_rn(acc.z, v.z);
            acc.w = __fadd_rn(acc.w, v.w);
        }
        __nv_bfloat16* o = y + 4 * i;
        o[0] = __float2bfloat16_rn(acc.x);
        o[1] = __float2bfloat16_rn(acc.y);
        o[2] = __float2bfloat16_rn(acc.z);
        o[3] = __float2bfloat16_rn(acc.w);
    }
}

cudaError_t launch_fp8_pack(int N, int K, const uint8_t* wq, const uint8_t* ws, void* packed, bool fwd,
                            uint8_t* out_wq, uint8_t* out_ws, cudaStream_t st) {
    uint8_t* p = (uint8_t*)packed;
    int32_t* flag = &reinterpret_cast<Fp8Header*>(p)->flag;
    if (fwd) {
        k_fp8_header<<<1, 1, 0, st>>>(p, N, K);
        count_launches(1);
    }
    const size_t pieces = (size_t)(N / 128) * (K / 128) * 1056;
    const int grid = (int)std::min<size_t>((pieces + 255) / 256, 148 * 16);
    k_fp8_pack<<<grid, 256, 0, st>>>(wq, ws, p + kFp8HeaderBytes, N, K, fwd, out_wq, out_ws, flag);
    count_launches(1);
    return cudaGetLastError();
}

static int fp8_grid() {
    static PerContext cache;
    return cache.get([] {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaFuncSetAttribute(k_fp8_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(F8Shared)) !=
                cudaSuccess)
            return -1;
        return sms;
    });
}

cudaError_t launch_fp8_linear(const void* x, int T, int N, int K, const void* packed, void* y, void* ws,
                              uint8_t* dbg_q, uint8_t* dbg_s, uint64_t wait_ns, cudaStream_t st) {
    int32_t* flag = (int32_t*)ws;
    uint8_t* xb = (uint8_t*)ws + 256;
    const size_t nb = (size_t)(T + F8_BN - 1) / F8_BN;
    uint8_t* xs = xb + nb * (K / 128) * F8_B_BYTES;
    cudaError_t e = launch_pdl(k_fp8_quant_act, dim3(T), dim3(256), 0, st, (const __nv_bfloat16*)x, T, K, xb, xs,
                               dbg_q, dbg_s, (const uint8_t*)packed, N, flag);
    count_launches(1);
    if (e != cudaSuccess) return e;
    const int grid = fp8_grid();
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    // split the K range when one token tile leaves most SMs without a tile
    const int RB = N / F8_BM, KG = K / 128;
    int S = 1;
    // (up to two items per CTA: its two pipes stream them at the same time)
    if (T <= kFp8SplitMaxT && RB < grid) S = std::max(1, std::min({2 * grid / RB, kFp8MaxSplits, KG}));
    float* part = (float*)((uint8_t*)ws + fp8_part_offset(T, K));
    F8Args a{(const uint8_t*)packed + kFp8HeaderBytes, xb, xs, T, N, K, (__nv_bfloat16*)y, flag, wait_ns, S, part};
    e = launch_pdl(k_fp8_gemm, dim3(grid), dim3(F8_THREADS), sizeof(F8Shared), st, a);
    count_launches(1);
    if (e != cudaSuccess || S == 1) return e;
    const size_t n4 = (size_t)T * N / 4;
    e = launch_pdl(k_fp8_reduce, dim3((unsigned)std::min<size_t>((n4 + 255) / 256, 148 * 8)), dim3(256), 0, st,
                   (const float*)part, S, T, N, (__nv_bfloat16*)y, (const int32_t*)flag);
    count_launches(1);
    return e;
}

}  // namespace moe
