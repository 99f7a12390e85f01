// Tensor-core grouped GEMM, token-major form (the default for prefill-size
// calls).
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) moves its prefill expert GEMMs
// onto matrix cores with better reuse of the packed weights.  This form runs
// the same exact sum as the weight-major kernel (tc_gemm.cu) with the operands
// the other way round, which halves the shared-memory traffic of the
// activations per unit of tensor-core work:
//
//   A (M = 128) = the digit planes of 128 sorted token rows of one expert (the
//       INT8 activations as three exact E2M1 planes, q = 64a + 8b + c, plane p
//       with the constant scale 2^(6 - 3p)); stage-major layout written by the
//       x-plane / requant kernels: per 128-input stage and 8-row group
//       [plane][32-input chunk][8 rows][16 bytes] = 1536 bytes, so the rows of
//       a tile form one contiguous block per stage: one bulk copy.
//   B (N = 128 per MMA) = one packed weight chunk (pack.cu: 512 scale bytes in
//       the tensor cores' 128 x 4 scale-factor atom, then 8 KB of codes in
//       no-swizzle K-major core-matrix order): one bulk copy per chunk.
//   D (TMEM, fp32; lane = token row, column = weight row) = sum over planes of
//       A * SFA * B * SFB = sum_k q * w, exact while partial sums stay below
//       2^24 units of the row's smallest weight scale.
//
// A tile is 128 token rows x 256 weight rows (two packed chunks).  Each stage
// holds the tile's A planes (24 KB) once and both weight chunks (2 x 8.5 KB):
// 41 KB for 12 MMAs of 128 x 128 x 64, against 33 KB for 6 such MMAs in the
// weight-major form.  Two MMA-issuer warps share every stage, one per weight
// chunk (an issuing warp sustains about one block-scaled MMA per 123 clocks,
// and a 128 x 128 x 64 FP4 MMA takes 64 clocks of tensor-core time, so one
// issuer per 128-column half keeps the tensor core busy).
//
// One persistent CTA per SM, warp-specialised:
//   warp 0       producer: three bulk copies per stage (A planes, two weight
//                chunks) into a 5-stage ring (mbarrier transaction counts);
//   warps 1, 2   MMA issuers, one per weight chunk of the tile: its scale
//                factors to TMEM (tcgen05.cp), 2 x 3 MMAs per stage, a
//                tcgen05.commit that frees the stage (the empty barrier counts
//                both issuers) and, after the last stage, publishes the tile;
//   warps 4..19  epilogue, one per (TMEM lane quadrant, 64-column group): the
//                accumulator is read into registers and released at once, then
//                W1 forms SwiGLU from the gate and up columns of each 32-row
//                weight group (row interleave of pack.cu) and writes fp32 h, W2
//                writes the final fp32 Y.  The accumulator is read in the
//                16-lane x 256-bit shape, in which four consecutive threads
//                hold eight consecutive columns of one token row, so every
//                store instruction writes whole 32-byte sectors of eight rows.
// Three 128-column accumulators rotate over the (tile, half) sequence: use
// u = 2j + h (half h of the CTA's tile j) takes accumulator u mod 3.  At a
// tile boundary the issuer of half 0 finds its accumulator long drained (it
// last held half 1 of the tile two back), and only the issuer of half 1 waits
// for the epilogue to read half 0 of the tile just finished, so the tensor
// core keeps working while a tile drains.  Every epilogue warp waits for every
// use in order and releases it (count 16), the warps of the other half without
// reading it: each barrier's phases are then seen one after another by all of
// its waiters, so no parity wait can mistake a phase two ahead or behind (an
// issuer waits for the release of use u - 3 only after it has seen the release
// of use u - 5, which every warp gave after that of u - 6).
// Every wait is bounded in time; a wait that gives up raises FLAG_TIMEOUT and
// the roles wind down (copies in flight are waited for, TMEM is freed).
#include "kernels.cuh"
#include "moe_common.cuh"
#include "tcgen05.cuh"

namespace moe {

namespace {

constexpr int TN_M = kTcTokenTile;                 // token rows per tile (MMA M)
constexpr int TN_HALF = kTcWeightTile;             // weight rows per packed chunk and per MMA (N)
constexpr int TN_BN = kTcTnWeightTile;             // weight rows per tile (two chunks)
constexpr int TN_CHUNK = 512 + kTcWeightTile * 64; // packed chunk: scale atom + 128 rows x 128 inputs
constexpr int TN_A_BYTES = TN_M / 8 * kPlaneGroupBytes;
constexpr int TN_STAGE_BYTES = TN_A_BYTES + 2 * TN_CHUNK;
constexpr int TN_EPI_WARP0 = 4;                    // warps 0..3: producer, two issuers, idle
constexpr int TN_EPI_WARPS = 16;
constexpr int TN_THREADS = 32 * (TN_EPI_WARP0 + TN_EPI_WARPS);
constexpr int TN_STAGES = 5;
constexpr int TN_ACC = 3;                          // 128-column accumulators
// TMEM columns: accumulator b at 128b; per issuer h the three constant plane
// scales (4 columns each) at TN_SFA_COL + 12h; per issuer h and stage s the
// weight scale factors at TN_SFB_COL + 4 (TN_STAGES h + s).
constexpr int TN_SFA_COL = TN_ACC * TN_HALF;
constexpr int TN_SFB_COL = TN_SFA_COL + 24;
constexpr int TN_TMEM_COLS = 512;
static_assert(TN_BN == 2 * TN_HALF, "a tile is two packed chunks");
static_assert(TN_SFB_COL + 2 * TN_STAGES * 4 <= TN_TMEM_COLS, "accumulators and scale factors exceed TMEM");
static_assert(TN_STAGE_BYTES % 16 == 0 && TN_A_BYTES % 16 == 0 && TN_CHUNK % 16 == 0, "bulk-copy alignment");

struct TnShared {
    uint8_t stage[TN_STAGES][TN_STAGE_BYTES];
    uint8_t sfa[3][512];   // constant plane scales 2^6, 2^3, 2^0 in the scale-factor atom layout
    uint64_t full[TN_STAGES], empty[TN_STAGES], acc_full[TN_ACC], acc_empty[TN_ACC], drain[2];
    uint32_t tmem_base;
    int32_t abort;
};
static_assert(sizeof(TnShared) <= 227 * 1024, "shared memory per CTA");

struct TnArgs {
    const uint8_t* w;          // matrix region of the packed buffer
    size_t expert_bytes;
    int K;                     // inputs per weight row
    int N;                     // weight rows per expert (a multiple of 128)
    int gate_up_half;          // W1: I (gate/up interleave), W2: 0
    const uint8_t* planes;     // digit planes, stage-major
    int plane_rows;            // rows of the plane buffer (multiple of 16)
    const int32_t* plane_off;  // [E+1] first plane row of each expert (multiple of 16)
    int P;                     // sorted rows (pairs)
    const int32_t* offsets;    // [E+1]
    const int32_t* tile_off;   // [E+1] exclusive scan of tiles per expert (token tiles x 256-row blocks)
    int E;
    int32_t* flag;
    const float* row_scale;    // activation scale per source row (W1: sx per token, W2: sh per sorted row)
    const int32_t* perm;       // sorted row -> pair id (W1: source row = perm[i] / k_div)
    int k_div;                 // W1: k; W2: 0 (source row = sorted row)
    float* out;                // W1: h [P, I]; W2: Y [P, H]  (fp32, final values)
    uint64_t wait_ns;          // limit of every bounded wait (global-timer nanoseconds)
    int withhold;              // timeout test: CTA 0 withholds its first stage
};

struct TnTile {
    int e, rb, halves, i0, pr0, n_valid, n_rows;   // rb: 256-row weight block; halves: its chunks (1 or 2)
};

__device__ __forceinline__ TnTile tn_tile_at(const TnArgs& a, int t) {
    int lo = 0, hi = a.E;  // last e with tile_off[e] <= t
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(a.tile_off + mid) <= t) lo = mid; else hi = mid;
    }
    TnTile tt;
    tt.e = lo;
    const int RB = (a.N + TN_BN - 1) / TN_BN;
    const int local = t - __ldg(a.tile_off + lo);
    const int nb = local / RB;
    tt.rb = local % RB;
    tt.halves = min(2, (a.N - tt.rb * TN_BN) / TN_HALF);
    const int r0 = __ldg(a.offsets + lo), r1 = __ldg(a.offsets + lo + 1);
    tt.i0 = r0 + nb * TN_M;
    tt.pr0 = __ldg(a.plane_off + lo) + nb * TN_M;
    tt.n_valid = min(TN_M, r1 - tt.i0);
    tt.n_rows = (tt.n_valid + 15) & ~15;
    return tt;
}

// Instruction descriptor of kind::mxf4 block-scaled MMA: E2M1 x E2M1, UE8M0
// scales, fp32 accumulate, both operands K-major, M = 128, N = 128, K = 64;
// b_sf_id selects the weight scales' byte pair of the K half.
__device__ __forceinline__ uint32_t tn_idesc(int b_sf_id) {
    uint32_t d = 0;
    d |= (uint32_t)(b_sf_id & 3) << 4;
    d |= 1u << 7;                               // A format: E2M1
    d |= 1u << 10;                              // B format: E2M1
    d |= (uint32_t)(TN_HALF >> 3) << 17;        // N / 8
    d |= 1u << 23;                              // scale format UE8M0
    d |= (uint32_t)(TN_M >> 4) << 24;           // M / 16
    return d;                                   // a_sf_id = 0: the plane scales are constant
}

// 16 TMEM lanes (from the lane in taddr) x 64 columns, without waiting.  Shape
// 16x256b, 8 repetitions: thread t receives, for repetition j (columns 8j ..
// 8j + 7), r[4j], r[4j+1] = lane t/4, columns 8j + 2(t%4) + {0, 1} and
// r[4j+2], r[4j+3] = lane 8 + t/4, the same columns.
__device__ __forceinline__ void tn_ld16x64(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tn_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(TN_THREADS, 1) k_tc_gemm_tn(TnArgs a) {
    pdl_begin();
    extern __shared__ __align__(1024) uint8_t tn_smem_raw[];
    TnShared& sh = *reinterpret_cast<TnShared*>(tn_smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KG = a.K / 128;
    const int total = __ldg(a.tile_off + a.E);
    if (*(volatile int32_t*)a.flag & FLAG_LAYOUT) return;
    // tiles t = blockIdx.x + j * gridDim.x, j < ntiles (uniform per CTA)
    const int ntiles = (int)blockIdx.x < total ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    if (ntiles == 0) return;
    auto tile_of = [&](int j) { return (int)blockIdx.x + j * (int)gridDim.x; };

    // ---- set-up: barriers, constant plane scales, TMEM ----
    if (threadIdx.x == 0) {
        for (int s = 0; s < TN_STAGES; ++s) {
            mbar_init(smem_u32(&sh.full[s]), 1);
            mbar_init(smem_u32(&sh.empty[s]), 2);   // both issuers' commits
        }
        for (int b = 0; b < TN_ACC; ++b) {
            mbar_init(smem_u32(&sh.acc_full[b]), 1);                  // one issuer's commit
            mbar_init(smem_u32(&sh.acc_empty[b]), TN_EPI_WARPS);      // every epilogue warp
        }
        mbar_init(smem_u32(&sh.drain[0]), 1);
        mbar_init(smem_u32(&sh.drain[1]), 1);
        sh.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = threadIdx.x; i < 3 * 512; i += TN_THREADS) sh.sfa[i / 512][i % 512] = (uint8_t)(133 - 3 * (i / 512));
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sh.tmem_base)),
                     "r"(TN_TMEM_COLS)
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
    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        return mbar_wait_for<false>(bar, parity, a.wait_ns, abort);
    };
    // the last waits before TMEM is freed ignore the abort flag; one that
    // still runs out raises FLAG_TIMEOUT (the call's results are then invalid)
    auto final_wait = [&](uint32_t bar, uint32_t parity) {
        if (!mbar_wait_for<false>(bar, parity, a.wait_ns, nullptr)) raise_flag(a.flag, FLAG_TIMEOUT);
    };

    if (warp == 0) {
        // ---------------- producer ----------------
        int stage = 0;
        uint32_t phase = 0;
        bool filled[TN_STAGES] = {};
        uint32_t fill_parity[TN_STAGES] = {};
        for (int j = 0; j < ntiles && !*abort; ++j) {
            const TnTile tt = tn_tile_at(a, tile_of(j));
            const uint8_t* wexp = a.w + (size_t)tt.e * a.expert_bytes;
            const uint32_t abytes = (uint32_t)(tt.n_rows / 8) * kPlaneGroupBytes;
            // the tile's rows must lie inside the plane buffer (a plane_off
            // table that did not come from the planner is refused here)
            const bool rows_ok = tt.pr0 >= 0 && (tt.pr0 & 15) == 0 && tt.pr0 + tt.n_rows <= a.plane_rows;
            if (!rows_ok && lane == 0) raise_flag(a.flag, FLAG_BOUNDS);
            for (int g = 0; g < KG; ++g) {
                const uint32_t fb = smem_u32(&sh.full[stage]), eb = smem_u32(&sh.empty[stage]);
                if (!wait(eb, phase ^ 1u)) {
                    give_up();
                    break;
                }
                const uint32_t sbase = smem_u32(sh.stage[stage]);
                // timeout test: CTA 0 issues neither the copies nor the arrival
                // of its first stage, so the issuers waiting for it run out of time
                const bool withheld = a.withhold && blockIdx.x == 0 && j == 0 && g == 0;
                if (lane == 0 && !withheld) {
                    if (rows_ok) {
                        mbar_expect_tx(fb, abytes + (uint32_t)tt.halves * TN_CHUNK);
                        bulk_g2s(sbase, a.planes + ((size_t)g * (a.plane_rows / 8) + tt.pr0 / 8) * kPlaneGroupBytes,
                                 abytes, fb);
                        for (int h = 0; h < tt.halves; ++h)
                            bulk_g2s(sbase + TN_A_BYTES + h * TN_CHUNK,
                                     wexp + ((size_t)(2 * tt.rb + h) * KG + g) * TN_CHUNK, TN_CHUNK, fb);
                    } else {
                        mbar_arrive(fb);  // keep the ring moving; the tile's result is not used
                    }
                }
                __syncwarp();
                filled[stage] = !withheld;
                fill_parity[stage] = phase;
                if (++stage == TN_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // let every copy this warp issued land before the CTA can exit
        for (int s = 0; s < TN_STAGES; ++s)
            if (filled[s] && lane == 0) final_wait(smem_u32(&sh.full[s]), fill_parity[s]);
        __syncwarp();
    } else if (warp <= 2) {
        // ---------------- MMA issuer of weight chunk h ----------------
        const int h = warp - 1;
        const uint32_t sfa_col = tmem + TN_SFA_COL + 12 * h;
        const uint32_t sfb_col = tmem + TN_SFB_COL + 4 * TN_STAGES * h;
        if (lane == 0)
            for (int p = 0; p < 3; ++p) tc_cp_sf(sfa_col + 4 * p, make_sdesc(smem_u32(sh.sfa[p]), 0, 128));
        __syncwarp();
        int stage = 0;
        uint32_t phase = 0;
        for (int j = 0; j < ntiles && !*abort; ++j) {
            const TnTile tt = tn_tile_at(a, tile_of(j));
            const bool active = h < tt.halves;
            // accumulator of (tile j, half h) and how often it was used before
            const int u = 2 * j + h, buf = u % TN_ACC;
            const uint32_t use = (uint32_t)(u / TN_ACC);
            const uint32_t dcol = tmem + buf * TN_HALF;
            if (!wait(smem_u32(&sh.acc_empty[buf]), (use & 1u) ^ 1u)) {
                give_up();
                break;
            }
            tc_fence_after();
            bool ok = true;
            for (int g = 0; g < KG; ++g) {
                if (!wait(smem_u32(&sh.full[stage]), phase)) {
                    give_up();
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    if (active) {
                        const uint32_t sa = smem_u32(sh.stage[stage]);
                        const uint32_t sb = sa + TN_A_BYTES + h * TN_CHUNK;
                        const uint32_t sfb = sfb_col + 4 * stage;
                        tc_cp_sf(sfb, make_sdesc(sb, 0, 128));
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {
                            // weights: K-adjacent core matrices 2048 bytes apart, 8-row groups 128 apart
                            const uint64_t bdesc = make_sdesc(sb + 512 + ks * 2 * 2048, 2048, 128);
#pragma unroll
                            for (int p = 0; p < 3; ++p) {
                                // plane p, chunks 2ks and 2ks+1: K-adjacent core matrices
                                // 128 bytes apart, 8-row groups 1536 apart
                                const uint64_t adesc = make_sdesc(sa + p * 512 + ks * 256, 128, kPlaneGroupBytes);
                                tc_mma_mxf4(dcol, adesc, bdesc, tn_idesc(2 * ks), sfa_col + 4 * p, sfb,
                                            (g | ks | p) != 0);
                            }
                        }
                    }
                    tc_commit(smem_u32(&sh.empty[stage]));
                }
                __syncwarp();
                if (++stage == TN_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            // (an issuer without a chunk in this tile publishes its accumulator
            // unchanged, which keeps the rotation's phases in step)
            if (lane == 0) tc_commit(smem_u32(&sh.acc_full[buf]));
            __syncwarp();
        }
        // before the CTA frees TMEM every MMA this warp issued must be done
        if (lane == 0) {
            tc_commit(smem_u32(&sh.drain[h]));
            final_wait(smem_u32(&sh.drain[h]), 0);
        }
        __syncwarp();
    } else if (warp >= TN_EPI_WARP0) {
        // ---------------- epilogue (warps TN_EPI_WARP0 ..) ----------------
        // Warp (q, c) owns token rows 32q .. 32q + 31 of every tile (TMEM lane
        // quadrant q) and the 64 weight columns 64c .. 64c + 63 of the tile
        // (half c / 2, columns 64 (c % 2) .. of that half's accumulator).
        // Thread t holds rows 32q + t/4 + 8k (k = 0..3) at columns
        // 8j + 2(t%4) + {0, 1} (j = 0..7) of the group.  Scaling: the
        // accumulator is an fp32 value, so fp32(fp64(s) * fp64(acc)) -- the
        // definition -- is the single correctly rounded fp32 product s * acc.
        const int ew = warp - TN_EPI_WARP0;
        const int q = warp & 3;          // TMEM lane quadrant this warp may access
        const int cg = ew >> 2;          // 64-column group of the tile
        const int half = cg >> 1;
        const int t4 = lane >> 2, c2 = 2 * (lane & 3);
        const bool w1 = a.gate_up_half > 0;
        // waits for use u and releases it (the caller reads it in between)
        auto acquire = [&](int u) -> bool {
            if (!wait(smem_u32(&sh.acc_full[u % TN_ACC]), (uint32_t)(u / TN_ACC) & 1u)) {
                give_up();
                return false;
            }
            tc_fence_after();
            return true;
        };
        auto release = [&](int u) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sh.acc_empty[u % TN_ACC]));
        };
        for (int j = 0; j < ntiles && !*abort; ++j) {
            const TnTile tt = tn_tile_at(a, tile_of(j));
            const bool mine = half < tt.halves;
            const int u = 2 * j + half, buf = u % TN_ACC;
            float s[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int m = 32 * q + t4 + 8 * k;
                s[k] = 0.0f;
                if (mine && m < tt.n_valid) {
                    const int i = tt.i0 + m;
                    const int src = a.k_div > 0 ? checked_index(__ldg(a.perm + i), a.P, a.flag) / a.k_div : i;
                    s[k] = __ldg(a.row_scale + src);
                }
            }
            // the other half's use of this tile, when it comes first
            if (half == 1) {
                if (!acquire(u - 1)) break;
                release(u - 1);
            }
            if (!acquire(u)) break;
            uint32_t v[64];   // v[32L + 4jj + 2hh + e]: row 32q + 16L + 8hh + t/4, column 8jj + c2 + e
            if (mine) {
                const uint32_t taddr =
                    tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * TN_HALF + (cg & 1) * 64);
                tn_ld16x64(taddr, v);
                tn_ld16x64(taddr + (16u << 16), v + 32);
                tn_wait_ld();
            }
            // the values are in registers: release the accumulator
            release(u);
            // the other half's use of this tile, when it comes second
            if (half == 0) {
                if (!acquire(u + 1)) break;
                release(u + 1);
            }
            if (!mine) continue;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int m = 32 * q + t4 + 8 * k;
                if (m >= tt.n_valid) continue;
                const int i = tt.i0 + m;
                const int L = k >> 1, hh = k & 1;
                const uint32_t* r = v + 32 * L + 2 * hh;
                if (!w1) {
                    float* out = a.out + (size_t)i * a.N + tt.rb * TN_BN + cg * 64 + c2;
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        *reinterpret_cast<float2*>(out + 8 * jj) =
                            make_float2(__fmul_rn(s[k], __uint_as_float(r[4 * jj])),
                                        __fmul_rn(s[k], __uint_as_float(r[4 * jj + 1])));
                } else {
                    // column groups jj = 4g + {0, 1} are the gate rows, 4g + {2, 3}
                    // the up rows of outputs 16 (global 32-row group) + 8 (jj % 4) + c2 + e
                    float* out = a.out + (size_t)i * a.gate_up_half + tt.rb * (TN_BN / 2) + cg * 32 + c2;
#pragma unroll
                    for (int g = 0; g < 2; ++g)
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const int jg = 4 * g + jj;
                            *reinterpret_cast<float2*>(out + 16 * g + 8 * jj) =
                                make_float2(swiglu(__fmul_rn(s[k], __uint_as_float(r[4 * jg])),
                                                   __fmul_rn(s[k], __uint_as_float(r[4 * (jg + 2)]))),
                                            swiglu(__fmul_rn(s[k], __uint_as_float(r[4 * jg + 1])),
                                                   __fmul_rn(s[k], __uint_as_float(r[4 * (jg + 2) + 1]))));
                        }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TN_TMEM_COLS) : "memory");
}

int tn_grid() {
    static PerContext cache;
    return cache.get([] {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaFuncSetAttribute(k_tc_gemm_tn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(TnShared)) !=
                cudaSuccess)
            return -1;
        return sms;
    });
}

}  // namespace

cudaError_t launch_tc_gemm_tn(const uint8_t* w, size_t expert_bytes, int K, int N, int gate_up_half,
                              const uint8_t* planes, int plane_rows, const int32_t* plane_off, int P,
                              const int32_t* offsets, const int32_t* tile_off, int E, int32_t* flag,
                              const float* row_scale, const int32_t* perm, int k_div, float* out, uint64_t wait_ns,
                              int withhold, cudaStream_t st) {
    if (N % TN_HALF != 0 || K % 128 != 0) return cudaErrorInvalidValue;
    TnArgs a{w, expert_bytes, K, N, gate_up_half, planes, plane_rows, plane_off, P, offsets, tile_off,
             E, flag, row_scale, perm, k_div, out, wait_ns, withhold};
    const int grid = tn_grid();
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    const cudaError_t e = launch_pdl(k_tc_gemm_tn, dim3(grid), dim3(TN_THREADS), sizeof(TnShared), st, a);
    count_launches(1);
    return e;
}

}  // namespace moe
