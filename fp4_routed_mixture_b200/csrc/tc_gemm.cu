// Tensor-core grouped GEMM for experts with many rows (prefill).
//
// "DeepSeek-V4-Flash on AMD gfx90a" (abstract) moves its prefill expert GEMMs
// onto matrix-core kernels with better reuse of the packed weights.  On B200
// the same step runs on the 5th-generation tensor cores with the FP4 weights
// consumed natively: tcgen05.mma kind::mxf4 with block scaling (E2M1 operands,
// one UE8M0 scale per 32 inputs), operands staged in shared memory by TMA bulk
// copies, accumulators in tensor memory.
//
// Operands (swap-AB: the weights take the 128-row M side, tokens the N side):
//   A = one 128-row block of an expert's weights; each 128-input group is one
//       packed chunk (pack.cu): 512 scale bytes in the tensor cores' 128 x 4
//       scale-factor atom, then 8 KB of codes in no-swizzle K-major
//       core-matrix order.  One bulk copy per chunk.
//   B = the INT8 activations of the expert's sorted rows, written exactly as
//       three E2M1 digit planes: q = 64*a + 8*b + c with a, b, c in [-4, 3]
//       (balanced base-8 digits; every digit is an E2M1 value).  Plane p has
//       the constant scale 2^(6 - 3p).  The planes are stored stage-major:
//       for every 128-input stage and group of 8 rows, [plane][32-input
//       chunk][8 rows][16 bytes] (1536 bytes), and every expert's rows start
//       on a 16-row boundary, so the whole B operand of a tile and stage is
//       one contiguous block: one bulk copy (the copy engine moves about one
//       copy per 80 clocks per CTA, so many small copies cannot feed the MMAs).
//   D (TMEM, fp32) = sum over planes of A * SFA * B_p * SFB_p = sum_k w * q:
//       the same exact sum the CUDA-core kernel forms (every product is an
//       integer multiple of the row's smallest weight scale).
//
// One persistent CTA per SM, warp-specialised, with two independent pipes
// that take alternate tiles of the CTA's share:
//   warps 0, 1   producers: two bulk copies per stage (A chunk, B planes)
//                into the pipe's own 3-stage ring (mbarrier transaction
//                counts);
//   warps 2, 3   MMA issuers: scale factors to TMEM (tcgen05.cp), 2 x 3 MMAs
//                per stage, tcgen05.commit frees the stage / publishes the
//                tile;
//   warps 4..19  epilogue, one per (TMEM lane quadrant, 32-column chunk),
//                tiles in order: TMEM -> registers (tcgen05.ld), one thread
//                per weight row; W1 applies the token scale and SwiGLU (gate
//                and up rows share a warp) and writes h, W2 writes the final
//                fp32 Y.
// Three 128-column accumulators in TMEM, tile j in buffer j % 3: two tiles
// take MMAs while the epilogue drains the third.  Why two issuers: the tensor
// core queues only a few MMAs, and a thread that waits on an mbarrier (a
// shared-memory operation, ordered behind its own queued MMAs) stalls for
// about as long as that queue lasts at N <= 128, so one issuer leaves the pipe
// idle about half the time; two fill each other's gaps (measured 62-65 clocks
// per 128 x 112..128 x 64 MMA per SM against 56-64 ideal, ~125 with one).  Why
// 128-row token tiles: an MMA with N below 128 costs about as much as one
// with N = 128, so fewer, fuller tiles win.
// Every wait is bounded in time; a wait that gives up raises FLAG_TIMEOUT and
// the roles wind down (copies in flight are waited for, TMEM is freed).
#include "kernels.cuh"
#include "moe_common.cuh"
#include "tcgen05.cuh"

namespace moe {

constexpr int TC_BM = kTcWeightTile;           // weight rows per tile (MMA M)
constexpr int TC_PIPES = 2;                    // producer + MMA-issuer pairs, alternating tiles
constexpr int TC_ACC = 3;                      // accumulator buffers shared by the pipes
constexpr int TC_A_BYTES = 8704;               // one packed chunk: 128 rows x 128 inputs
constexpr int TC_EPI_WARP0 = 2 * TC_PIPES;     // warps 0..: producers, then MMA issuers

constexpr int pow2_at_least(int v, int p = 32) { return p >= v ? p : pow2_at_least(v, 2 * p); }

// A kernel configuration: BN token rows per tile (the largest MMA N used) and
// STAGES ring stages per pipe.  The prefill form takes 128-row token tiles
// with three 33 KB stages per pipe; the decode form (at most a few rows per
// expert) takes 32-row tiles with six 14.5 KB stages per pipe, which keeps
// twice the weight bytes in flight per SM -- at decode sizes the weights
// stream from DRAM and every byte is used by one tile.
template <int BN_, int STAGES_>
struct TcCfg {
    static constexpr int BN = BN_, STAGES = STAGES_;
    static constexpr int B_BYTES = BN / 8 * kPlaneGroupBytes;  // 3 planes x BN rows x 128 inputs
    static constexpr int STAGE_BYTES = TC_A_BYTES + B_BYTES;
    static constexpr int CHUNKS = BN / 32;                      // 32-column chunks of a tile
    static constexpr int EPI_WARPS = 4 * CHUNKS;                // one per (TMEM lane quadrant, column chunk)
    static constexpr int THREADS = 32 * (TC_EPI_WARP0 + EPI_WARPS);
    // TMEM columns: accumulator b at b * BN; then per pipe r, at SF_COL +
    // SF_PIPE_COLS * r, the A scale factors (4 columns per stage) and the three
    // constant B plane scales (4 columns each).
    static constexpr int SF_COL = TC_ACC * BN;
    static constexpr int SF_PIPE_COLS = 4 * STAGES + 12;
    // The A-in-TMEM form (ATMEM): every stage's weight chunk is copied into
    // TMEM once (tcgen05.cp, two 128 x 256-bit halves, 16 columns) and the six
    // plane MMAs read A from there, so shared memory feeds only B.  Columns:
    // the accumulators, then per pipe r and stage s the A slot at AT_A +
    // 16 (STAGES r + s), the A scale factors at AT_SFA + 4 (STAGES r + s), and
    // two constant B scale regions shared by the pipes: X (bytes 2^6, 2^6, 2^3,
    // 2^3 in every 4-byte group) serves planes 0 and 1 through the
    // scale-factor byte selector (0 and 2), Y (all 2^0) plane 2.
    static constexpr int AT_A = TC_ACC * BN;
    static constexpr int AT_SFA = AT_A + TC_PIPES * STAGES * 16;
    static constexpr int AT_SFB = AT_SFA + TC_PIPES * STAGES * 4;
    static constexpr int TMEM_COLS = pow2_at_least(
        (SF_COL + TC_PIPES * SF_PIPE_COLS) > (AT_SFB + 8) ? (SF_COL + TC_PIPES * SF_PIPE_COLS) : (AT_SFB + 8));
    static_assert(TMEM_COLS <= 512, "accumulators, A slots and scale factors exceed TMEM");
    static_assert(SF_COL % 4 == 0 && SF_PIPE_COLS % 4 == 0, "scale-factor columns hold 4 bytes per lane");
    static_assert(AT_A % 16 == 0, "A slots on 16-column boundaries");
    static_assert(BN % 32 == 0 && BN <= 256, "MMA N, whole column chunks");

    struct Shared {
        uint8_t stage[TC_PIPES][STAGES][STAGE_BYTES];
        uint8_t sfb[3][512];        // constant plane scales, copied to TMEM by the MMA issuers
        float col_scale[EPI_WARPS][32];  // per epilogue warp: activation scale of its 32 columns
        uint64_t full[TC_PIPES][STAGES], empty[TC_PIPES][STAGES], acc_full[TC_ACC], acc_empty[TC_ACC];
        uint64_t drain[TC_PIPES];   // each issuer's last commit: all of its MMAs are done
        uint64_t sfb_ready;         // ATMEM: the shared B scale regions are in TMEM
        uint32_t tmem_base;
        int32_t abort;
    };
};
using TcPrefill = TcCfg<kTcTokenTile, 3>;
using TcDecode = TcCfg<kTcDecodeTokenTile, 6>;
static_assert(sizeof(TcPrefill::Shared) <= 227 * 1024 && sizeof(TcDecode::Shared) <= 227 * 1024,
              "shared memory per CTA");

struct TcArgs {
    const uint8_t* w;          // matrix region of the packed buffer
    size_t expert_bytes;
    int K;                     // inputs per weight row
    int N;                     // weight rows per expert
    int gate_up_half;          // W1: I (gate/up interleave), W2: 0
    const uint8_t* planes;     // digit planes, stage-major (see above)
    int plane_rows;            // rows of the plane buffer (multiple of 16)
    const int32_t* plane_off;  // [E+1] first plane row of each expert (multiple of 16)
    int P;                     // sorted rows (pairs)
    const int32_t* offsets;    // [E+1]
    const int32_t* tile_off;   // [E+1] exclusive scan of tiles per expert
    int E;
    int32_t* flag;
    // epilogue
    const float* row_scale;    // activation scale per source row (W1: sx per token, W2: sh per sorted row)
    const int32_t* perm;       // sorted row -> pair id (W1: source row = perm[i] / k_div)
    int k_div;                 // W1: k; W2: 0 (source row = sorted row)
    float* out;                // W1: h [P, I]; W2: Y [P, H]  (fp32, final values)
    uint64_t wait_ns;          // limit of every bounded wait (global-timer nanoseconds)
    int withhold;              // test of the timeout path: 1 = see launch_tc_gemm
};

// ---- the SM-pair form (cta_group::2) ----------------------------------------
// Two CTAs of a cluster share one MMA: the even CTA issues it with M = 256; each
// CTA supplies its own 128 weight rows (A) and half of the token rows (B) from
// the same shared-memory offsets, and each CTA's TMEM receives the accumulator
// rows of its own weight rows.
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void mbar_arrive_peer(uint32_t bar, uint32_t rank) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(peer_addr(bar, rank))
                 : "memory");
}
__device__ __forceinline__ void store_peer_u32(uint32_t addr, uint32_t rank, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_addr(addr, rank)), "r"(v) : "memory");
}
// tcgen05.commit of the pair's MMAs, arriving on the barrier at this offset in
// both CTAs.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"((uint16_t)3)
        : "memory");
}
__device__ __forceinline__ void tc_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_mma_mxf4_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                                 uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Instruction descriptor of kind::mxf4 block-scaled MMA: E2M1 x E2M1, UE8M0
// scales, fp32 accumulate, both operands K-major, M = 128, K = 64.
template <int M = TC_BM>
__device__ __forceinline__ uint32_t make_idesc(int n, int a_sf_id, int b_sf_id) {
    uint32_t d = 0;
    d |= (uint32_t)(b_sf_id & 3) << 4;
    d |= 1u << 7;                          // A format: E2M1
    d |= 1u << 10;                         // B format: E2M1
    d |= (uint32_t)(n >> 3) << 17;         // N / 8
    d |= 1u << 23;                         // scale format UE8M0
    d |= (uint32_t)(M >> 4) << 24;         // M / 16 (the pair form: 256)
    d |= (uint32_t)(a_sf_id & 3) << 29;
    return d;
}

struct TcTile {
    int e, rb, i0, pr0, n_valid, n_mma;   // i0: first sorted row, pr0: its plane row
};

template <int TC_BN>
__device__ __forceinline__ TcTile tile_at(const TcArgs& a, int t) {
    int lo = 0, hi = a.E;  // last e with tile_off[e] <= t
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(a.tile_off + mid) <= t) lo = mid; else hi = mid;
    }
    TcTile tt;
    tt.e = lo;
    const int RB = a.N / TC_BM;
    const int local = t - __ldg(a.tile_off + lo);
    const int nb = local / RB;
    tt.rb = local % RB;
    const int r0 = __ldg(a.offsets + lo), r1 = __ldg(a.offsets + lo + 1);
    tt.i0 = r0 + nb * TC_BN;
    tt.pr0 = __ldg(a.plane_off + lo) + nb * TC_BN;
    tt.n_valid = min(TC_BN, r1 - tt.i0);
    tt.n_mma = (tt.n_valid + 15) & ~15;
    return tt;
}

// PAIR = false: one CTA per SM, 128-row tiles.  PAIR = true: clusters of two
// CTAs; the pair takes the adjacent 128-row tiles 2m (even CTA) and 2m + 1
// (odd CTA) of one expert and token tile and computes them with M = 256 MMAs
// issued by the even CTA.  Each CTA loads its own A chunk and half of the
// tile's token rows (B), so a stage moves 8.7 KB + 12.3 KB into each SM
// instead of 8.7 KB + 24.6 KB.  Roles in the pair: the odd CTA's MMA warps
// relay "stage landed" to the even CTA (its copies complete on its own
// barrier; a remote arrive joins the even CTA's), the even CTA's MMA commits
// arrive on the barriers of both CTAs, and the odd CTA's epilogue warps release
// accumulators with remote arrives.
template <class Cfg, bool PAIR, bool ATMEM>
__global__ void __launch_bounds__(Cfg::THREADS, 1) k_tc_gemm(TcArgs a) {
    static_assert(!(PAIR && ATMEM), "the A-in-TMEM form is one CTA per SM");
    constexpr int TC_BN = Cfg::BN, TC_STAGES = Cfg::STAGES, TC_EPI_WARPS = Cfg::EPI_WARPS;
    constexpr int TC_THREADS = Cfg::THREADS, TC_TMEM_COLS = Cfg::TMEM_COLS;
    constexpr int TC_SF_COL = Cfg::SF_COL, TC_SF_PIPE_COLS = Cfg::SF_PIPE_COLS;
    constexpr int TC_AT_A = Cfg::AT_A, TC_AT_SFA = Cfg::AT_SFA, TC_AT_SFB = Cfg::AT_SFB;
    using TcShared = typename Cfg::Shared;
    pdl_begin();
    extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
    TcShared& sh = *reinterpret_cast<TcShared*>(tc_smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KG = a.K / 128;
    const int total = __ldg(a.tile_off + a.E);
    // (both CTAs of a pair read the same values, so they leave together)
    if (*(volatile int32_t*)a.flag & FLAG_LAYOUT) return;
    if (total == 0) return;
    const uint32_t rank = PAIR ? cluster_rank() : 0u, peer = rank ^ 1u;
    const bool leader = rank == 0;
    // work units: tiles (PAIR: pairs of tiles), unit u_j = unit0 + j * nunits,
    // j < ntiles; unit j belongs to pipe j % TC_PIPES and accumulator j % TC_ACC
    const int unit0 = PAIR ? (int)blockIdx.x >> 1 : (int)blockIdx.x;
    const int nunits = PAIR ? (int)gridDim.x >> 1 : (int)gridDim.x;
    const int units = PAIR ? total / 2 : total;
    const int ntiles = unit0 < units ? (units - unit0 + nunits - 1) / nunits : 0;
    auto tile_of = [&](int j) { return PAIR ? 2 * (unit0 + j * nunits) + (int)rank : unit0 + j * nunits; };

    // ---- set-up: barriers, constant plane scales, TMEM ----
    if (threadIdx.x == 0) {
        for (int r = 0; r < TC_PIPES; ++r)
            for (int s = 0; s < TC_STAGES; ++s) {
                // the even CTA of a pair also waits for the odd CTA's relay
                mbar_init(smem_u32(&sh.full[r][s]), PAIR && leader ? 2 : 1);
                mbar_init(smem_u32(&sh.empty[r][s]), 1);
            }
        for (int b = 0; b < TC_ACC; ++b) {
            mbar_init(smem_u32(&sh.acc_full[b]), 1);
            mbar_init(smem_u32(&sh.acc_empty[b]), PAIR ? 2 * TC_EPI_WARPS : TC_EPI_WARPS);
        }
        for (int r = 0; r < TC_PIPES; ++r) mbar_init(smem_u32(&sh.drain[r]), 1);
        mbar_init(smem_u32(&sh.sfb_ready), 1);
        sh.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = threadIdx.x; i < 3 * 512; i += TC_THREADS) {
        const int p = i / 512;
        if (ATMEM)  // regions X (2^6, 2^6, 2^3, 2^3 per 4 bytes) and Y (2^0)
            sh.sfb[p][i % 512] = (uint8_t)(p == 0 ? ((i & 3) < 2 ? 133 : 130) : 127);
        else
            sh.sfb[p][i % 512] = (uint8_t)(133 - 3 * p);  // 2^6, 2^3, 2^0
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 0) {
        if (PAIR) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(&sh.tmem_base)),
                         "r"(TC_TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_u32(&sh.tmem_base)),
                         "r"(TC_TMEM_COLS)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();  // the peer's barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    volatile int32_t* abort = &sh.abort;
    auto give_up = [&]() {
        *abort = 1;
        if (PAIR) store_peer_u32(smem_u32(&sh.abort), peer, 1u);
        raise_flag(a.flag, FLAG_TIMEOUT);
    };
    // bounded waits; barriers that pair operations arrive on are read at
    // cluster scope
    auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
        return mbar_wait_for<PAIR>(bar, parity, a.wait_ns, abort);
    };
    // the last waits before TMEM is freed ignore the abort flag: a wait that
    // still runs out raises FLAG_TIMEOUT (the caller must then treat the whole
    // call's results as invalid; the CTA still frees TMEM and exits)
    auto final_wait = [&](uint32_t bar, uint32_t parity) {
        if (!mbar_wait_for<PAIR>(bar, parity, a.wait_ns, nullptr)) raise_flag(a.flag, FLAG_TIMEOUT);
    };

    if (warp < TC_PIPES) {
        // ---------------- producer of pipe r ----------------
        const int r = warp;
        int stage = 0;
        uint32_t phase = 0;
        bool filled[TC_STAGES] = {};
        uint32_t fill_parity[TC_STAGES] = {};
        for (int j = r; j < ntiles && !*abort; j += TC_PIPES) {
            const TcTile tt = tile_at<TC_BN>(a, tile_of(j));
            const uint8_t* wsrc = a.w + (size_t)tt.e * a.expert_bytes + (size_t)tt.rb * KG * TC_A_BYTES;
            // token rows this CTA supplies: all of them, or its half of the pair's
            const int nb_rows = PAIR ? tt.n_mma / 2 : tt.n_mma;
            const int b_row0 = tt.pr0 + (PAIR ? (int)rank * nb_rows : 0);
            const uint32_t bbytes = (uint32_t)(nb_rows / 8) * kPlaneGroupBytes;  // B of one stage
            // the tile's rows must lie inside the plane buffer (a plane_off
            // table that did not come from the planner is refused here)
            const bool rows_ok = tt.pr0 >= 0 && (tt.pr0 & 15) == 0 && tt.pr0 + tt.n_mma <= a.plane_rows;
            if (!rows_ok && lane == 0) raise_flag(a.flag, FLAG_BOUNDS);
            for (int g = 0; g < KG; ++g) {
                const uint32_t fb = smem_u32(&sh.full[r][stage]), eb = smem_u32(&sh.empty[r][stage]);
                if (!wait(eb, phase ^ 1u)) {
                    give_up();
                    break;
                }
                const uint32_t sbase = smem_u32(sh.stage[r][stage]);
                // timeout test: CTA 0's first producer issues neither the copies
                // nor the arrival of its first stage, so the MMA issuer waiting
                // for that stage runs out of time
                const bool withheld = !PAIR && a.withhold && blockIdx.x == 0 && r == 0 && j == 0 && g == 0;
                if (lane == 0 && !withheld) {
                    if (rows_ok) {
                        mbar_expect_tx(fb, TC_A_BYTES + bbytes);
                        bulk_g2s(sbase, wsrc + (size_t)g * TC_A_BYTES, TC_A_BYTES, fb);
                        const uint8_t* src =
                            a.planes + ((size_t)g * (a.plane_rows / 8) + b_row0 / 8) * kPlaneGroupBytes;
                        bulk_g2s(sbase + TC_A_BYTES, src, bbytes, fb);
                    } else {
                        mbar_arrive(fb);  // keep the ring moving; the tile's result is not used
                    }
                }
                __syncwarp();
                filled[stage] = !withheld;
                fill_parity[stage] = phase;
                if (++stage == TC_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // let every copy this warp issued land before the CTA can exit (on the
        // normal path the MMA warp has already waited for all of them)
        for (int s = 0; s < TC_STAGES; ++s)
            if (filled[s] && lane == 0) final_wait(smem_u32(&sh.full[r][s]), fill_parity[s]);
        __syncwarp();
    } else if (warp < TC_EPI_WARP0 && PAIR && !leader) {
        // ---------------- relay of pipe r (odd CTA of a pair) ----------------
        // Passes "this CTA's half of the stage has landed" to the even CTA,
        // stage by stage in the producer's order, then waits for the pair's
        // last MMAs (they write this CTA's TMEM) before the CTA may free it.
        const int r = warp - TC_PIPES;
        int stage = 0;
        uint32_t phase = 0;
        for (int j = r; j < ntiles && !*abort; j += TC_PIPES) {
            bool ok = true;
            for (int g = 0; g < KG; ++g) {
                if (!wait(smem_u32(&sh.full[r][stage]), phase)) {
                    give_up();
                    ok = false;
                    break;
                }
                if (lane == 0) mbar_arrive_peer(smem_u32(&sh.full[r][stage]), peer);
                __syncwarp();
                if (++stage == TC_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
        }
        if (lane == 0 && ntiles > r) final_wait(smem_u32(&sh.drain[r]), 0);
        __syncwarp();
    } else if (warp < TC_EPI_WARP0) {
        // ---------------- MMA issuer of pipe r (even CTA of a pair) ----------------
        const int r = warp - TC_PIPES;
        const uint32_t sfa_col = ATMEM ? tmem + TC_AT_SFA + 4 * TC_STAGES * r : tmem + TC_SF_COL + TC_SF_PIPE_COLS * r;
        const uint32_t sfb_col = ATMEM ? tmem + TC_AT_SFB : sfa_col + 4 * TC_STAGES;
        const uint32_t a_col = tmem + TC_AT_A + 16 * TC_STAGES * r;
        bool sfb_ok = true;
        if (ATMEM) {
            // pipe 0 copies the two shared B scale regions; pipe 1 waits for them
            if (lane == 0) {
                if (r == 0) {
                    tc_cp_sf(sfb_col, make_sdesc(smem_u32(sh.sfb[0]), 0, 128));
                    tc_cp_sf(sfb_col + 4, make_sdesc(smem_u32(sh.sfb[1]), 0, 128));
                    tc_commit(smem_u32(&sh.sfb_ready));
                } else {
                    sfb_ok = wait(smem_u32(&sh.sfb_ready), 0);
                }
            }
            sfb_ok = __shfl_sync(0xffffffffu, sfb_ok, 0);
            if (!sfb_ok) give_up();
            tc_fence_after();
        } else if (lane == 0) {
            for (int p = 0; p < 3; ++p) {
                if (PAIR)
                    tc_cp_sf_pair(sfb_col + 4 * p, make_sdesc(smem_u32(sh.sfb[p]), 0, 128));
                else
                    tc_cp_sf(sfb_col + 4 * p, make_sdesc(smem_u32(sh.sfb[p]), 0, 128));
            }
        }
        __syncwarp();
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        for (int j = r; j < ntiles && sfb_ok && !*abort; j += TC_PIPES) {
            const TcTile tt = tile_at<TC_BN>(a, tile_of(j));
            const int buf = j % TC_ACC;
            const uint32_t use = (uint32_t)(j / TC_ACC);
            if (!wait(smem_u32(&sh.acc_empty[buf]), (use & 1u) ^ 1u)) {
                give_up();
                break;
            }
            tc_fence_after();
            const uint32_t dcol = tmem + buf * TC_BN;
            bool ok = true;
            for (int g = 0; g < KG; ++g) {
                if (!wait(smem_u32(&sh.full[r][stage]), phase)) {
                    give_up();
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t sbase = smem_u32(sh.stage[r][stage]);
                    const uint32_t sfa = sfa_col + 4 * stage;
                    if (PAIR)
                        tc_cp_sf_pair(sfa, make_sdesc(sbase, 0, 128));
                    else
                        tc_cp_sf(sfa, make_sdesc(sbase, 0, 128));
                    if (ATMEM) {
                        // the stage's A into its TMEM slot, once for all six MMAs
                        // (the slot is rewritten only after this stage's MMAs
                        // have completed: the producer refills the stage after
                        // their commit)
                        const uint32_t at = a_col + 16 * stage;
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks)
                            tc_cp_a(at + 8 * ks, make_sdesc(sbase + 512 + ks * 2 * 2048, 2048, 128));
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                            for (int p = 0; p < 3; ++p) {
                                const uint64_t bdesc = make_sdesc(sbase + TC_A_BYTES + p * 512 + ks * 256, 128,
                                                                  kPlaneGroupBytes);
                                // planes 0 and 1: region X, bytes 0-1 / 2-3; plane 2: region Y
                                tc_mma_mxf4_at(dcol, at + 8 * ks, bdesc,
                                               make_idesc(tt.n_mma, 2 * ks, p == 1 ? 2 : 0), sfa,
                                               sfb_col + (p == 2 ? 4 : 0), (g | ks | p) != 0);
                            }
                    }
#pragma unroll
                    for (int ks = 0; ks < (ATMEM ? 0 : 2); ++ks) {
                        const uint64_t adesc = make_sdesc(sbase + 512 + ks * 2 * 2048, 2048, 128);
#pragma unroll
                        for (int p = 0; p < 3; ++p) {
                            // plane p, chunks 2ks and 2ks+1: K-adjacent core
                            // matrices 128 bytes apart, 8-row groups 1536 apart
                            const uint64_t bdesc = make_sdesc(sbase + TC_A_BYTES + p * 512 + ks * 256, 128,
                                                              kPlaneGroupBytes);
                            if (PAIR)
                                tc_mma_mxf4_pair(dcol, adesc, bdesc, make_idesc<2 * TC_BM>(tt.n_mma, 2 * ks, 0), sfa,
                                                 sfb_col + 4 * p, (g | ks | p) != 0);
                            else
                                tc_mma_mxf4(dcol, adesc, bdesc, make_idesc(tt.n_mma, 2 * ks, 0), sfa,
                                            sfb_col + 4 * p, (g | ks | p) != 0);
                        }
                    }
                    if (PAIR)
                        tc_commit_pair(smem_u32(&sh.empty[r][stage]));
                    else
                        tc_commit(smem_u32(&sh.empty[r][stage]));
                }
                __syncwarp();
                if (++stage == TC_STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) {
                if (PAIR)
                    tc_commit_pair(smem_u32(&sh.acc_full[buf]));
                else
                    tc_commit(smem_u32(&sh.acc_full[buf]));
            }
            __syncwarp();
            ++issued;
        }
        // before the CTA frees TMEM, every MMA this warp issued must be done
        // (on the normal path the epilogue has already seen them finish; after a
        // timeout some may still be in flight).  In a pair the commit also
        // reaches the odd CTA, whose relay waits for it.
        if (lane == 0) {
            if (PAIR) {
                if (ntiles > r) {
                    tc_commit_pair(smem_u32(&sh.drain[r]));
                    final_wait(smem_u32(&sh.drain[r]), 0);
                }
            } else {
                tc_commit(smem_u32(&sh.drain[r]));
                final_wait(smem_u32(&sh.drain[r]), 0);
            }
        }
        (void)issued;
        __syncwarp();
    } else {
        // ---------------- epilogue (warps TC_EPI_WARP0 ..) ----------------
        // Warp (q, c) owns the 32 weight rows of TMEM lane quadrant q and the
        // 32-column chunk c of every tile, tiles in this CTA's order.  It first
        // stages the activation scale of its columns in its own shared-memory
        // slice (no cross-warp waits).  Scaling: the accumulator is an fp32
        // value, so fp32(fp64(s) * fp64(acc)) -- the definition -- equals the
        // single correctly rounded fp32 product s * acc (the exact product of
        // two 24-bit significands fits in fp64).
        // W1: lanes 0-15 of a warp hold the gate rows and lanes 16-31 the up
        // rows of the same 16 outputs (row interleave of pack.cu).  Columns go
        // in pairs: lanes 0-15 form h for column j (up value shuffled down),
        // lanes 16-31 for column j+1 (gate value shuffled up), h = SwiGLU(g, u),
        // stored in fp32 (the row maximum of |h| is taken when h is
        // requantised).  W2: Y = s * acc straight out.  In a pair each CTA
        // drains its own tile (its TMEM holds its weight rows); the odd CTA
        // releases the accumulator to the even CTA's MMA warps remotely.
        const int ew = warp - TC_EPI_WARP0;
        const int q = warp & 3;            // TMEM lane quadrant this warp may access
        const int n0 = 32 * (ew >> 2);     // this warp's column chunk
        const int m = q * 32 + lane;       // weight row within the tile
        const bool w1 = a.gate_up_half > 0;
        float* csc = sh.col_scale[ew];
        for (int j = 0; j < ntiles && !*abort; ++j) {
            const TcTile tt = tile_at<TC_BN>(a, tile_of(j));
            const int buf = j % TC_ACC;
            const uint32_t use = (uint32_t)(j / TC_ACC);
            const bool mine = n0 < tt.n_mma;
            if (mine) {
                const int i = min(tt.i0 + n0 + lane, tt.i0 + tt.n_valid - 1);
                const int src = a.k_div > 0 ? checked_index(__ldg(a.perm + i), a.P, a.flag) / a.k_div : i;
                csc[lane] = __ldg(a.row_scale + src);
            }
            __syncwarp();
            if (!wait(smem_u32(&sh.acc_full[buf]), use & 1u)) {
                give_up();
                break;
            }
            tc_fence_after();
            if (mine) {
                uint32_t v[32];
                tc_ld32(tmem + ((uint32_t)(q * 32) << 16) + buf * TC_BN + n0, v);
                if (!w1) {
                    float* out = a.out + (size_t)(tt.i0 + n0) * a.N + tt.rb * TC_BM + m;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (n0 + c < tt.n_valid) out[(size_t)c * a.N] = __fmul_rn(csc[c], __uint_as_float(v[c]));
                } else {
                    const int I = a.gate_up_half;
                    const bool lo = lane < 16;
                    float* out = a.out + (size_t)(tt.i0 + n0) * I + (tt.rb * 4 + q) * 16 + (lane & 15);
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float v0 = __fmul_rn(csc[c], __uint_as_float(v[c]));
                        const float v1 = __fmul_rn(csc[c + 1], __uint_as_float(v[c + 1]));
                        const float from_hi = __shfl_down_sync(0xffffffffu, v0, 16);  // up value, column c
                        const float from_lo = __shfl_up_sync(0xffffffffu, v1, 16);    // gate value, column c+1
                        const float hv = lo ? swiglu(v0, from_hi) : swiglu(from_lo, v1);
                        if (n0 + c + (lo ? 0 : 1) < tt.n_valid) out[(size_t)(c + (lo ? 0 : 1)) * I] = hv;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (PAIR && !leader)
                    mbar_arrive_peer(smem_u32(&sh.acc_empty[buf]), peer);
                else
                    mbar_arrive(smem_u32(&sh.acc_empty[buf]));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();  // no remote arrive or MMA targets this CTA any more
    tc_fence_after();
    if (warp == 0) {
        if (PAIR)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_TMEM_COLS)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_TMEM_COLS)
                         : "memory");
    }
}

// Copies the x digit planes of every sorted row of a tensor-core expert from
// token order (k_xquant: per token and 32-input block c, 48 bytes = plane p's
// 16 bytes at +16p) into the stage-major layout: plane p, block c = 4*g + cc of
// plane row pr -> 16 bytes at planes + (g*(plane_rows/8) + pr/8)*1536 + p*512
// + cc*128 + (pr%8)*16.  Source token of sorted row i: perm[i] / k_div; its
// plane row is plane_row[i] (-1: a row of a streaming-GEMM expert, skipped).
// One thread per (row, block), rows fastest: 8 consecutive rows fill 128
// contiguous bytes of each plane.  Grid: (rows / 256, K / 128); a thread
// copies the 4 blocks of one stage of its row.
__global__ void __launch_bounds__(256)
    k_planes(const uint8_t* __restrict__ tplanes, int K, const int32_t* __restrict__ perm, int k_div, int rows,
             const int32_t* __restrict__ plane_row, int plane_rows, uint8_t* __restrict__ planes,
             int32_t* flag) {
    pdl_begin();
    const int nc = K / 32;
    const int i = blockIdx.x * blockDim.x + threadIdx.x, g = blockIdx.y;
    if (i >= rows) return;
    const int pr = __ldg(plane_row + i);
    if (pr < 0) return;
    if (pr >= plane_rows) {
        raise_flag(flag, FLAG_BOUNDS);
        return;
    }
    const int t = checked_index(__ldg(perm + i), rows, flag) / k_div;
    const uint4* s = reinterpret_cast<const uint4*>(tplanes + ((size_t)t * nc + 4 * g) * 48);
    uint4 v[12];
#pragma unroll
    for (int u = 0; u < 12; ++u) v[u] = __ldg(s + u);   // blocks 4g..4g+3, planes 0..2
    uint8_t* dst = planes + ((size_t)g * (plane_rows / 8) + (pr >> 3)) * kPlaneGroupBytes + (pr & 7) * 16;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int p = 0; p < 3; ++p) *reinterpret_cast<uint4*>(dst + p * 512 + cc * 128) = v[3 * cc + p];
}

// One CTA per SM (it allocates the SM's TMEM) for every form of the kernel:
// sets the dynamic shared-memory limit of each one-CTA instantiation.
template <class Cfg>
static cudaError_t set_smem(void (*k)(TcArgs)) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(typename Cfg::Shared));
}

static int tc_grid() {
    static PerContext cache;
    return cache.get([] {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            set_smem<TcPrefill>(k_tc_gemm<TcPrefill, false, false>) != cudaSuccess ||
            set_smem<TcPrefill>(k_tc_gemm<TcPrefill, false, true>) != cudaSuccess ||
            set_smem<TcDecode>(k_tc_gemm<TcDecode, false, false>) != cudaSuccess ||
            set_smem<TcDecode>(k_tc_gemm<TcDecode, false, true>) != cudaSuccess)
            return -1;
        return sms;
    });
}

// Clusters of two CTAs that can be resident at once (0: the pair form is not
// available); the grid is two CTAs per such cluster, so no cluster waits for
// another to finish.  (The pair form is built for the prefill configuration.)
static int tc_pair_grid() {
    static PerContext cache;
    return cache.get([] {
        const int single = tc_grid();
        if (single <= 0) return -1;
        if (set_smem<TcPrefill>(k_tc_gemm<TcPrefill, true, false>) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * single);
        cfg.blockDim = dim3(TcPrefill::THREADS);
        cfg.dynamicSmemBytes = sizeof(TcPrefill::Shared);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, k_tc_gemm<TcPrefill, true, false>, &cfg) != cudaSuccess ||
            clusters <= 0) {
            cudaGetLastError();
            return 0;
        }
        return 2 * clusters;
    });
}

size_t tc_smem_bytes() { return sizeof(TcPrefill::Shared); }

cudaError_t launch_planes(const uint8_t* tplanes, int K, const int32_t* perm, int k_div, int rows,
                          const int32_t* plane_row, int plane_rows, uint8_t* planes, int32_t* flag,
                          cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    const cudaError_t e = launch_pdl(k_planes, dim3((unsigned)((rows + 255) / 256), (unsigned)(K / 128)),
                                     dim3(256), 0, st, tplanes, K, perm, k_div, rows, plane_row, plane_rows, planes,
                                     flag);
    count_launches(1);
    return e;
}

cudaError_t launch_tc_gemm(const uint8_t* w, size_t expert_bytes, int K, int N, int gate_up_half,
                           const uint8_t* planes, int plane_rows, const int32_t* plane_off, int P,
                           const int32_t* offsets, const int32_t* tile_off, int E, int32_t* flag,
                           const float* row_scale, const int32_t* perm, int k_div, float* out, int token_tile,
                           bool pair, bool a_tmem, uint64_t wait_ns, int withhold, cudaStream_t st) {
    TcArgs a{w, expert_bytes, K, N, gate_up_half, planes, plane_rows, plane_off, P, offsets, tile_off,
             E, flag, row_scale, perm, k_div, out, wait_ns, withhold};
    const bool decode = token_tile == TcDecode::BN;
    if (!decode && token_tile != TcPrefill::BN) return cudaErrorInvalidValue;
    // the timeout test runs on the one-CTA form (withhold applies to it only);
    // the A-in-TMEM and decode forms are one CTA per SM
    if (withhold || a_tmem || decode) pair = false;
    cudaError_t e;
    // the pair takes two adjacent 128-row tiles of one expert: N % 256 == 0
    const int pgrid = (pair && N % (2 * TC_BM) == 0) ? tc_pair_grid() : 0;
    if (pgrid > 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(pgrid);
        cfg.blockDim = dim3(TcPrefill::THREADS);
        cfg.dynamicSmemBytes = sizeof(TcPrefill::Shared);
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, k_tc_gemm<TcPrefill, true, false>, a);
    } else {
        const int grid = tc_grid();
        if (grid <= 0) return cudaErrorInvalidConfiguration;
        if (decode)
            e = a_tmem ? launch_pdl(k_tc_gemm<TcDecode, false, true>, dim3(grid), dim3(TcDecode::THREADS),
                                    sizeof(TcDecode::Shared), st, a)
                       : launch_pdl(k_tc_gemm<TcDecode, false, false>, dim3(grid), dim3(TcDecode::THREADS),
                                    sizeof(TcDecode::Shared), st, a);
        else
            e = a_tmem ? launch_pdl(k_tc_gemm<TcPrefill, false, true>, dim3(grid), dim3(TcPrefill::THREADS),
                                    sizeof(TcPrefill::Shared), st, a)
                       : launch_pdl(k_tc_gemm<TcPrefill, false, false>, dim3(grid), dim3(TcPrefill::THREADS),
                                    sizeof(TcPrefill::Shared), st, a);
    }
    count_launches(1);
    return e;
}

}  // namespace moe
