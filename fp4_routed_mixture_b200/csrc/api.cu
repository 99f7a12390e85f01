// C-ABI layer: argument checks, workspace layout, launch sequence.
// Declarations and the meaning of every argument are in include/moe.h.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstddef>
#include <cstdio>
#include <cstring>
#include <string>

#include "../../include/moe.h"
#include "kernels.cuh"
#include "moe_common.cuh"

#include <atomic>

namespace moe {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
}  // namespace moe

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* where) {
    return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int check_dims(const moe_dims* d, bool need_T) {
    if (!d) return fail(MOE_ERR_INVALID_ARG, "dims is NULL");
    if (need_T && d->T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0 (got %d)", d->T);
    if (d->H <= 0 || d->I <= 0 || d->H % 128 || d->I % 128)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "H and I must be positive multiples of 128 (H=%d I=%d)",
                    d->H, d->I);
    if (d->E < 1 || d->E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E must be in [1, 1024] (got %d)", d->E);
    if (d->k < 1 || d->k > 16 || d->k > d->E)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "k must be in [1, min(E, 16)] (got %d)", d->k);
    if (need_T && (long long)d->T * d->k >= (1LL << 31))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "T*k must be < 2^31");
    return MOE_OK;
}

// Process-wide options (moe_set_option).  Every public call reads them once
// into an Options value, so a call sees one consistent set even while another
// host thread changes them.
std::atomic<int> g_tc_min_rows{0};         // tensor-core row threshold; 0 = automatic (see tc_threshold)
std::atomic<int> g_tc_pair{0};             // tensor-core GEMM in SM pairs (cta_group::2) where the shape allows
std::atomic<int> g_wait_limit_us{1000000}; // limit of the tensor-core GEMM's bounded waits
std::atomic<int> g_test_timeout{0};        // one-shot: the next tensor-core launch withholds a stage
std::atomic<int> g_tc_a_tmem{0};           // tensor-core GEMM with the weight operand staged in TMEM
std::atomic<int> g_tc_form{0};             // forms of the prefill tensor-core GEMMs (MOE_OPT_TC_FORM)

struct Options {
    int tc_min_rows;
    bool tc_pair;
    bool tc_a_tmem;
    int tc_form;
    uint64_t wait_ns;
};

// The tensor-core row threshold of a call of T tokens.  Automatic (option 0):
// calls of fewer than kAutoTcMinT tokens run every expert on the streaming
// GEMM (with the fused front), larger calls put every expert with at least
// two rows on the tensor cores -- measured faster than the streaming GEMM from
// two rows up at decode_T64 and on the skewed prefill, while one-row experts
// stream better.  An explicit option value is used as it is.
constexpr int kAutoTcMinT = 32;
constexpr int kAutoTcMinRows = 2;
int tc_threshold(int option_value, long long T) {
    if (option_value > 0) return option_value;
    return T < kAutoTcMinT ? 0x7fffffff : kAutoTcMinRows;
}

Options load_options() {
    return Options{g_tc_min_rows.load(), g_tc_pair.load() != 0, g_tc_a_tmem.load() != 0,
                   g_tc_form.load(), 1000ull * (uint64_t)g_wait_limit_us.load()};
}

struct WsLayout {
    size_t flag, uoff1, uoff2, toff1, toff2, poff, soff, etc, prow, sx, xq, xtp, xinit, hq, sh, hinit, px, ph,
        hbuf, yf, gacc, yacc, total;
    int plane_rows;
    int stream_rows;   // capacity of the buffers of streaming-GEMM rows
};

// Rows the streaming GEMM can own in a call of T tokens: every row when no
// expert can reach the tensor-core threshold (T < tc_min), otherwise at most
// tc_min - 1 rows of each of the E experts.
long long stream_row_capacity(const moe_dims& d, long long T, int tc_min) {
    const long long P = T * d.k;
    if (T < tc_min) return P;
    return std::min(P, (long long)d.E * (tc_min - 1));
}

WsLayout ws_layout(const moe_dims& d, long long T, int tc_min) {
    using moe::align_up;
    const size_t P = (size_t)T * d.k;
    const size_t S = (size_t)stream_row_capacity(d, T, tc_min);
    WsLayout L;
    size_t o = 0;
    L.flag = o; o += 256;
    L.uoff1 = o; o += align_up(4 * (size_t)(d.E + 1), 256);
    L.uoff2 = o; o += align_up(4 * (size_t)(d.E + 1), 256);
    L.toff1 = o; o += align_up(4 * (size_t)(d.E + 1), 256);
    L.toff2 = o; o += align_up(4 * (size_t)(d.E + 1), 256);
    L.poff = o; o += align_up(4 * (size_t)(d.E + 1), 256);
    L.soff = o; o += align_up(4 * (size_t)(d.E + 1), 256);
    L.etc = o; o += align_up(4 * (size_t)d.E, 256);
    L.prow = o; o += align_up(4 * P, 256);
    L.sx = o; o += align_up(4 * (size_t)T, 256);
    L.xq = o; o += align_up((size_t)T * d.H, 256);
    L.xtp = o; o += align_up((size_t)T * (d.H / 32) * 48, 256);   // x digit planes, token order
    L.xinit = o; o += align_up(4 * (size_t)T * (d.H / 32), 256);
    L.stream_rows = (int)S;
    L.hq = o; o += align_up(S * d.I, 256);                  // h codes of streaming rows
    L.sh = o; o += align_up(4 * P, 256);
    L.hinit = o; o += align_up(4 * S * (d.I / 32), 256);
    // digit planes of the tensor-core GEMM (stage-major, see kernels.cuh):
    // each tensor-core expert's rows are padded to a multiple of 16
    L.plane_rows = (int)align_up(P + 16 * (size_t)d.E + 16, 16);
    L.px = o; o += align_up(moe::plane_bytes(d.H, L.plane_rows), 256);
    L.ph = o; o += align_up(moe::plane_bytes(d.I, L.plane_rows), 256);
    L.hbuf = o; o += align_up(4 * P * d.I, 256);        // h of every row (fp32)
    L.yf = o; o += align_up(4 * P * d.H, 256);          // Y of tensor-core rows
    L.gacc = o; o += align_up(8 * S * 2 * d.I, 256);   // fp64 sums of streaming-GEMM rows
    L.yacc = o; o += align_up(8 * S * d.H, 256);
    L.total = o;
    return L;
}

}  // namespace

extern "C" {

size_t moe_last_error(char* buf, size_t n) {
    if (buf && n) {
        const size_t c = std::min(n - 1, g_last_error.size());
        std::memcpy(buf, g_last_error.data(), c);
        buf[c] = 0;
    }
    return g_last_error.size();
}

size_t moe_packed_bytes(const moe_dims* d) {
    if (check_dims(d, false) != MOE_OK) return 0;
    return moe::packed_layout(d->H, d->I, d->E).total;
}

int moe_pack_weights(const moe_dims* d, const uint8_t* w1_codes, const uint8_t* w1_scales,
                     const uint8_t* w2_codes, const uint8_t* w2_scales, void* packed,
                     cudaStream_t stream) {
    g_last_error.clear();
    if (int rc = check_dims(d, false)) return rc;
    if (!w1_codes || !w1_scales || !w2_codes || !w2_scales || !packed)
        return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: NULL pointer");
    if (!aligned(w1_codes, 16) || !aligned(w2_codes, 16) || !aligned(packed, 256))
        return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: codes need 16-byte, packed 256-byte alignment");
    cudaError_t e = moe::launch_pack(d->H, d->I, d->E, w1_codes, w1_scales, w2_codes, w2_scales,
                                     packed, true, nullptr, nullptr, nullptr, nullptr, stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_pack_weights launch");
    int32_t flag = 0;
    e = cudaMemcpyAsync(&flag, moe::packed_flag_ptr(packed), sizeof(flag), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_pack_weights");
    if (flag & MOE_FLAG_BAD_SCALE)
        return fail(MOE_ERR_INVALID_ARG, "moe_pack_weights: scale byte 0xFF (E8M0 NaN) in the input");
    return MOE_OK;
}

int moe_unpack_weights(const moe_dims* d, const void* packed, uint8_t* w1_codes, uint8_t* w1_scales,
                       uint8_t* w2_codes, uint8_t* w2_scales, cudaStream_t stream) {
    g_last_error.clear();
    if (int rc = check_dims(d, false)) return rc;
    if (!w1_codes || !w1_scales || !w2_codes || !w2_scales || !packed)
        return fail(MOE_ERR_INVALID_ARG, "moe_unpack_weights: NULL pointer");
    if (!aligned(w1_codes, 16) || !aligned(w2_codes, 16) || !aligned(packed, 256))
        return fail(MOE_ERR_INVALID_ARG, "moe_unpack_weights: codes need 16-byte, packed 256-byte alignment");
    cudaError_t e = moe::launch_pack(d->H, d->I, d->E, nullptr, nullptr, nullptr, nullptr,
                                     const_cast<void*>(packed), false, w1_codes, w1_scales, w2_codes,
                                     w2_scales, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_unpack_weights launch");
}

int moe_router_logits(const void* x_bf16, const float* w_router, const float* bias, int T, int H, int E,
                      float* logits, cudaStream_t stream) {
    g_last_error.clear();
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "moe_router_logits: T < 0");
    if (H <= 0 || H % 32) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_router_logits: H must be a positive multiple of 32");
    if (E < 1 || E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_router_logits: E must be in [1, 1024]");
    if ((long long)T * H >= (1LL << 40) || (long long)T * E >= (1LL << 31))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_router_logits: T too large");
    if (T > 0 && (!x_bf16 || !w_router || !logits)) return fail(MOE_ERR_INVALID_ARG, "moe_router_logits: NULL pointer");
    if (!aligned(x_bf16, 16) || !aligned(w_router, 16))
        return fail(MOE_ERR_INVALID_ARG, "moe_router_logits: x and w_router need 16-byte alignment");
    cudaError_t e = moe::launch_router_logits(x_bf16, w_router, bias, T, H, E, logits, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_router_logits launch");
}

int moe_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* gates,
              cudaStream_t stream) {
    g_last_error.clear();
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "moe_route: T < 0");
    if (E < 1 || E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_route: E must be in [1, 1024]");
    if (k < 1 || k > 16 || k > E) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_route: k must be in [1, min(E,16)]");
    if (T > 0 && (!logits || !topk_idx || !gates)) return fail(MOE_ERR_INVALID_ARG, "moe_route: NULL pointer");
    cudaError_t e = moe::launch_route(logits, T, E, k, topk_idx, gates, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route launch");
}

size_t moe_sort_workspace_bytes(int T_max, int k, int E) {
    if (T_max < 0 || k < 1 || E < 1) return 0;
    return moe::sort_workspace_bytes(T_max, k, E);
}

int moe_sort(const int32_t* topk_idx, int T, int k, int E, int32_t* perm, int32_t* pos,
             int32_t* offsets, void* ws, size_t ws_bytes, cudaStream_t stream) {
    g_last_error.clear();
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "moe_sort: T < 0");
    if (E < 1 || E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_sort: E must be in [1, 1024]");
    if (k < 1 || k > 16 || k > E) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_sort: k must be in [1, min(E,16)]");
    if ((long long)T * k >= (1LL << 31)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_sort: T*k too large");
    if (!offsets || !ws || (T > 0 && (!topk_idx || !perm || !pos)))
        return fail(MOE_ERR_INVALID_ARG, "moe_sort: NULL pointer");
    if (!aligned(ws, 256)) return fail(MOE_ERR_INVALID_ARG, "moe_sort: ws must be 256-byte aligned");
    if (ws_bytes < moe::sort_workspace_bytes(T, k, E))
        return fail(MOE_ERR_INVALID_ARG, "moe_sort: ws_bytes %zu < %zu", ws_bytes,
                    moe::sort_workspace_bytes(T, k, E));
    cudaError_t e = moe::launch_sort(topk_idx, T, k, E, perm, pos, offsets, ws, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_sort launch");
}

int moe_sort_static(const int32_t* topk_idx, int T, int k, int E, int32_t* perm, int32_t* pos,
                    int32_t* offsets, cudaStream_t stream) {
    g_last_error.clear();
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "moe_sort_static: T < 0");
    if (E < 1 || E > 1024) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_sort_static: E must be in [1, 1024]");
    if (k < 1 || k > 16 || k > E)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_sort_static: k must be in [1, min(E,16)]");
    if (!moe::sort_static_fits(T, k, E))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "moe_sort_static: T*k = %lld exceeds the static scratch limit of 65536 pairs "
                    "(use moe_sort with a caller workspace)", (long long)T * k);
    if (!offsets || (T > 0 && (!topk_idx || !perm || !pos)))
        return fail(MOE_ERR_INVALID_ARG, "moe_sort_static: NULL pointer");
    cudaError_t e = moe::launch_sort_static(topk_idx, T, k, E, perm, pos, offsets, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_sort_static");
}

size_t moe_workspace_bytes(const moe_dims* d, int T_max) {
    if (check_dims(d, false) != MOE_OK || T_max < 0) return 0;
    const int v = g_tc_min_rows.load();
    size_t total = ws_layout(*d, T_max, tc_threshold(v, T_max)).total;
    // (automatic threshold: a call just below kAutoTcMinT tokens keeps every
    // row on the streaming GEMM and may need more than the larger T_max)
    if (v == 0 && T_max >= kAutoTcMinT)
        total = std::max(total, ws_layout(*d, kAutoTcMinT - 1, tc_threshold(v, kAutoTcMinT - 1)).total);
    return total;
}

}  // extern "C"

namespace {

// The layer from its routing tables on.  With logits == NULL, topk_idx, gates,
// perm, pos and offsets are inputs (moe_forward).  With logits != NULL
// (moe_layer_forward on a call with T below the tensor-core threshold and at
// most kFrontMaxPairs pairs) route, sort, x quant and plan run as one fused
// launch that writes those tables.
int forward_impl(const Options& opt, const moe_dims* d, const float* logits, const void* x_bf16, int32_t* topk_idx,
                 float* gates, int32_t* perm, int32_t* pos, int32_t* offsets, const void* packed, void* y_bf16,
                 void* ws, size_t ws_bytes, int32_t* flag_word, const moe_debug* dbg, cudaStream_t stream) {
    if (int rc = check_dims(d, true)) return rc;
    if (!ws || !packed || !offsets) return fail(MOE_ERR_INVALID_ARG, "moe_forward: NULL pointer");
    if (d->T > 0 && (!x_bf16 || !topk_idx || !gates || !perm || !pos || !y_bf16))
        return fail(MOE_ERR_INVALID_ARG, "moe_forward: NULL pointer");
    if (!aligned(ws, 256) || !aligned(packed, 256) || !aligned(x_bf16, 16) || !aligned(y_bf16, 16))
        return fail(MOE_ERR_INVALID_ARG, "moe_forward: ws/packed need 256-byte, x/y 16-byte alignment");
    const int tc_min = tc_threshold(opt.tc_min_rows, d->T);
    const WsLayout L = ws_layout(*d, d->T, tc_min);
    if (ws_bytes < L.total)
        return fail(MOE_ERR_INVALID_ARG,
                    "moe_forward: ws_bytes %zu < %zu (the size depends on MOE_OPT_TC_MIN_ROWS: size the "
                    "workspace after setting it)", ws_bytes, L.total);
    char* w = (char*)ws;
    int32_t* flag = flag_word ? flag_word : (int32_t*)(w + L.flag);
    if (d->T == 0) {  // no kernel runs; otherwise the first kernel clears the word
        cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(int32_t), stream);
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_forward memset");
    }

    const int T = d->T, H = d->H, I = d->I, E = d->E, k = d->k, P = T * k;
    const moe::PackedLayout PL = moe::packed_layout(H, I, E);
    const uint8_t* pk = (const uint8_t*)packed;
    int32_t* uoff1 = (int32_t*)(w + L.uoff1);
    int32_t* uoff2 = (int32_t*)(w + L.uoff2);
    float* sx = (float*)(w + L.sx);
    int8_t* xq = (int8_t*)(w + L.xq);
    int32_t* xinit = (int32_t*)(w + L.xinit);
    int8_t* hq = (int8_t*)(w + L.hq);
    float* sh = (float*)(w + L.sh);
    int32_t* hinit = (int32_t*)(w + L.hinit);
    double* gacc = (double*)(w + L.gacc);
    double* yacc = (double*)(w + L.yacc);

#define MOE_TRY(call, what)                          \
    do {                                             \
        cudaError_t _e = (call);                     \
        if (_e != cudaSuccess) return cuda_fail(_e, what); \
    } while (0)
    // an expert has at most T rows, so the tensor-core path is skipped without
    // reading any count when T < tc_min (always so with the fused front)
    const bool use_tc = !logits && T >= tc_min;
    // the timeout test applies to the first tensor-core launch after it is armed
    const int withhold = use_tc ? g_test_timeout.exchange(0) : 0;
    // Forms of the tensor-core GEMMs: W1 token-major (128 token rows x 256
    // weight rows per tile: half the activation-operand traffic per MMA), W2
    // weight-major (lanes are weight rows, so its fp32 Y rows are stored in
    // whole 128-byte lines) with 128-row token tiles, or 32-row ones (the
    // decode configuration) when no expert can have more than kTcDecodeMaxT
    // rows.  MOE_OPT_TC_FORM 1 / 2 take both weight-major / both token-major;
    // the weight-major variants (pair, A in TMEM) take both weight-major.
    const int wm_tile = T <= moe::kTcDecodeMaxT ? moe::kTcDecodeTokenTile : moe::kTcTokenTile;
    const bool wm_variant = opt.tc_pair || opt.tc_a_tmem;
    const bool tc_tn1 = !wm_variant && opt.tc_form != 1;
    const bool tc_tn2 = !wm_variant && opt.tc_form == 2;
    const int tc_tile1 = tc_tn1 ? moe::kTcTokenTile : wm_tile;
    const int tc_tile2 = tc_tn2 ? moe::kTcTokenTile : wm_tile;
    const int tc_wtile1 = tc_tn1 ? moe::kTcTnWeightTile : moe::kTcWeightTile;
    const int tc_wtile2 = tc_tn2 ? moe::kTcTnWeightTile : moe::kTcWeightTile;
    // with a threshold of 1 every expert with rows takes the tensor cores, so
    // the streaming GEMM has nothing to do and is not launched
    const bool use_gemv = !use_tc || tc_min > 1;
    // token rows per streaming-GEMM unit: 2 for small calls (nearly every expert
    // has one or two rows; the smaller ring slot fits more warps per SM), else 4
    const int group = T <= moe::kGemvSmallGroupMaxT ? moe::kGemvSmallGroup : moe::kGemvGroup;
    uint8_t* xtp = (uint8_t*)(w + L.xtp);
    int32_t* toff1 = (int32_t*)(w + L.toff1);
    int32_t* toff2 = (int32_t*)(w + L.toff2);
    uint8_t* px = (uint8_t*)(w + L.px);
    uint8_t* ph = (uint8_t*)(w + L.ph);
    int32_t* poff = (int32_t*)(w + L.poff);
    int32_t* soff = (int32_t*)(w + L.soff);
    int32_t* prow = (int32_t*)(w + L.prow);
    int32_t* etc = (int32_t*)(w + L.etc);
    float* hbuf = (float*)(w + L.hbuf);
    float* yf = (float*)(w + L.yf);
    if (logits) {
        MOE_TRY(moe::launch_layer_front(logits, x_bf16, packed, T, H, I, E, k, group, topk_idx, gates, perm, pos,
                                        offsets,
                                        uoff1, uoff2, prow, xq, sx, xinit,
                                        dbg ? dbg->xq : nullptr, dbg ? dbg->sx : nullptr, gacc, yacc, flag,
                                        stream),
                "route + sort + x quant + plan");
    } else {
        MOE_TRY(moe::launch_xquant(x_bf16, T, H, xq, sx, xinit, use_tc ? xtp : nullptr, dbg ? dbg->xq : nullptr,
                                   dbg ? dbg->sx : nullptr, packed, I, E, flag, stream),
                "x quant + header check");
        MOE_TRY(moe::launch_plan_rows(offsets, topk_idx, perm, E, P, I, H, use_tc ? tc_min : 0x7fffffff, tc_tile1,
                                      tc_tile2, tc_wtile1, tc_wtile2, group, uoff1, uoff2, toff1, toff2, poff, soff,
                                      etc, prow, gacc, yacc, flag, stream),
                "plan + row state");
    }
    if (use_tc)
        MOE_TRY(moe::launch_planes(xtp, H, perm, k, P, prow, L.plane_rows, px, flag, stream), "x planes");
    cudaEvent_t* ev = dbg ? const_cast<cudaEvent_t*>(dbg->events) : nullptr;
    if (ev && ev[0]) MOE_TRY(cudaEventRecord(ev[0], stream), "event");
    // (with the fused front every row is a streaming row: its streaming rows
    // are the sorted offsets)
    const int32_t* gemv_soff = logits ? offsets : soff;
    if (use_gemv)
        MOE_TRY(moe::launch_gemv(pk + PL.w1, PL.w1_expert_bytes, H, 2 * I, xq, xinit, perm, k, offsets,
                                 uoff1, gemv_soff, E, gacc, flag, I, P, group, false, stream), "W1");
    if (use_tc && tc_tn1)
        MOE_TRY(moe::launch_tc_gemm_tn(pk + PL.w1, PL.w1_expert_bytes, H, 2 * I, I, px, L.plane_rows, poff, P,
                                       offsets, toff1, E, flag, sx, perm, k, hbuf, opt.wait_ns, withhold, stream),
                "W1 tensor cores");
    else if (use_tc)
        MOE_TRY(moe::launch_tc_gemm(pk + PL.w1, PL.w1_expert_bytes, H, 2 * I, I, px, L.plane_rows, poff, P,
                                    offsets, toff1, E, flag, sx, perm, k, hbuf, tc_tile1, opt.tc_pair, opt.tc_a_tmem,
                                    opt.wait_ns, withhold, stream),
                "W1 tensor cores");
    if (ev && ev[1]) MOE_TRY(cudaEventRecord(ev[1], stream), "event");
    MOE_TRY(moe::launch_hquant(gacc, hbuf, sx, perm, prow, L.plane_rows, L.stream_rows, ph, P, k, I, hq, sh,
                               hinit, dbg ? dbg->hq : nullptr, dbg ? dbg->sh : nullptr, flag, stream),
            "SwiGLU + h quant + h planes");
    if (ev && ev[2]) MOE_TRY(cudaEventRecord(ev[2], stream), "event");
    if (use_gemv)
        MOE_TRY(moe::launch_gemv(pk + PL.w2, PL.w2_expert_bytes, I, H, hq, hinit, perm, 0, offsets,
                                 uoff2, gemv_soff, E, yacc, flag, 0, P, group, true, stream), "W2");
    if (use_tc && tc_tn2)
        MOE_TRY(moe::launch_tc_gemm_tn(pk + PL.w2, PL.w2_expert_bytes, I, H, 0, ph, L.plane_rows, poff, P,
                                       offsets, toff2, E, flag, sh, perm, 0, yf, opt.wait_ns, 0, stream),
                "W2 tensor cores");
    else if (use_tc)
        MOE_TRY(moe::launch_tc_gemm(pk + PL.w2, PL.w2_expert_bytes, I, H, 0, ph, L.plane_rows, poff, P,
                                    offsets, toff2, E, flag, sh, perm, 0, yf, tc_tile2, opt.tc_pair, opt.tc_a_tmem,
                                    opt.wait_ns, 0, stream),
                "W2 tensor cores");
    if (ev && ev[3]) MOE_TRY(cudaEventRecord(ev[3], stream), "event");
    MOE_TRY(moe::launch_combine(yacc, yf, logits ? nullptr : etc, offsets, soff, topk_idx, E, L.stream_rows, sh, gates,
                                pos, T, k, H, y_bf16, flag, stream),
            "combine");
#undef MOE_TRY
    return MOE_OK;
}

}  // namespace

extern "C" {

int moe_forward(const moe_dims* d, const void* x_bf16, const int32_t* topk_idx, const float* gates,
                const int32_t* perm, const int32_t* pos, const int32_t* offsets, const void* packed,
                void* y_bf16, void* ws, size_t ws_bytes, const moe_debug* dbg, cudaStream_t stream) {
    g_last_error.clear();
    return forward_impl(load_options(), d, nullptr, x_bf16, const_cast<int32_t*>(topk_idx), const_cast<float*>(gates),
                        const_cast<int32_t*>(perm), const_cast<int32_t*>(pos), const_cast<int32_t*>(offsets),
                        packed, y_bf16, ws, ws_bytes, nullptr, dbg, stream);
}

// Whole-layer workspace: the call's device error word, then
// idx/gates/perm/pos/offsets and the sort scratch (their offsets depend on T,
// k and E only, so moe_layer_tables needs no option), then the forward
// workspace (whose own error-word slot is not used: the layer's kernels report
// into the word at offset 0).
struct LayerWs {
    size_t flag, fwd, idx, gates, perm, pos, offsets, sortws, sort_bytes, total;
};

static LayerWs layer_ws(const moe_dims& d, long long T, int tc_min) {
    using moe::align_up;
    LayerWs L;
    const size_t P = (size_t)T * d.k;
    size_t o = 0;
    L.flag = o; o += 256;
    L.idx = o; o += align_up(4 * P, 256);
    L.gates = o; o += align_up(4 * P, 256);
    L.perm = o; o += align_up(4 * P, 256);
    L.pos = o; o += align_up(4 * P, 256);
    L.offsets = o; o += align_up(4 * (size_t)(d.E + 1), 256);
    L.sortws = o;
    L.sort_bytes = moe::sort_workspace_bytes((int)T, d.k, d.E);
    o += align_up(L.sort_bytes, 256);
    L.fwd = o; o += ws_layout(d, T, tc_min).total;
    L.total = o;
    return L;
}

size_t moe_layer_workspace_bytes(const moe_dims* d, int T_max) {
    if (check_dims(d, false) != MOE_OK || T_max < 0) return 0;
    const int v = g_tc_min_rows.load();
    size_t total = layer_ws(*d, T_max, tc_threshold(v, T_max)).total;
    if (v == 0 && T_max >= kAutoTcMinT)
        total = std::max(total, layer_ws(*d, kAutoTcMinT - 1, tc_threshold(v, kAutoTcMinT - 1)).total);
    return total;
}

int moe_layer_forward(const moe_dims* d, const float* logits, const void* x_bf16, const void* packed,
                      void* y_bf16, void* ws, size_t ws_bytes, const moe_debug* dbg,
                      cudaStream_t stream) {
    g_last_error.clear();
    if (int rc = check_dims(d, true)) return rc;
    if (!ws || !packed || (d->T > 0 && (!logits || !x_bf16 || !y_bf16)))
        return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: NULL pointer");
    if (!aligned(ws, 256)) return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward: ws must be 256-byte aligned");
    const Options opt = load_options();
    const int tc_min = tc_threshold(opt.tc_min_rows, d->T);
    const LayerWs L = layer_ws(*d, d->T, tc_min);
    if (ws_bytes < L.total)
        return fail(MOE_ERR_INVALID_ARG,
                    "moe_layer_forward: ws_bytes %zu < %zu (the size depends on MOE_OPT_TC_MIN_ROWS: size the "
                    "workspace after setting it)", ws_bytes, L.total);
    char* w = (char*)ws;
    int32_t* idx = (int32_t*)(w + L.idx);
    float* gates = (float*)(w + L.gates);
    int32_t* perm = (int32_t*)(w + L.perm);
    int32_t* pos = (int32_t*)(w + L.pos);
    int32_t* offsets = (int32_t*)(w + L.offsets);
    if (d->T > 0 && d->T < tc_min && (long long)d->T * d->k <= moe::kFrontMaxPairs)
        return forward_impl(opt, d, logits, x_bf16, idx, gates, perm, pos, offsets, packed, y_bf16, w + L.fwd,
                            L.total - L.fwd, (int32_t*)(w + L.flag), dbg, stream);
    if (int rc = moe_route(logits, d->T, d->E, d->k, idx, gates, stream)) return rc;
    if (int rc = moe_sort(idx, d->T, d->k, d->E, perm, pos, offsets, w + L.sortws, L.sort_bytes, stream))
        return rc;
    return forward_impl(opt, d, nullptr, x_bf16, idx, gates, perm, pos, offsets, packed, y_bf16, w + L.fwd,
                        L.total - L.fwd, (int32_t*)(w + L.flag), dbg, stream);
}

// moe_layer_forward preceded by the router projection: the logits go to a
// region after the layer workspace.
static size_t router_ws_offset(const moe_dims& d, long long T, int tc_min) {
    return moe::align_up(layer_ws(d, T, tc_min).total, 256);
}

size_t moe_layer_router_workspace_bytes(const moe_dims* d, int T_max) {
    if (check_dims(d, false) != MOE_OK || T_max < 0) return 0;
    return moe::align_up(moe_layer_workspace_bytes(d, T_max), 256) + moe::align_up(4 * (size_t)T_max * d->E, 256);
}

int moe_layer_forward_with_router(const moe_dims* d, const void* x_bf16, const float* w_router,
                                  const float* bias, const void* packed, void* y_bf16, void* ws,
                                  size_t ws_bytes, const moe_debug* dbg, cudaStream_t stream) {
    g_last_error.clear();
    if (int rc = check_dims(d, true)) return rc;
    if (!ws || !packed || (d->T > 0 && (!x_bf16 || !w_router || !y_bf16)))
        return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward_with_router: NULL pointer");
    if (!aligned(ws, 256))
        return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward_with_router: ws must be 256-byte aligned");
    const size_t lo = router_ws_offset(*d, d->T, tc_threshold(g_tc_min_rows.load(), d->T));
    const size_t need = lo + moe::align_up(4 * (size_t)d->T * d->E, 256);
    if (ws_bytes < need)
        return fail(MOE_ERR_INVALID_ARG, "moe_layer_forward_with_router: ws_bytes %zu < %zu", ws_bytes, need);
    float* logits = (float*)((char*)ws + lo);
    if (int rc = moe_router_logits(x_bf16, w_router, bias, d->T, d->H, d->E, logits, stream)) return rc;
    return moe_layer_forward(d, logits, x_bf16, packed, y_bf16, ws, lo, dbg, stream);
}

int moe_layer_tables(const moe_dims* d, void* ws, int32_t** topk_idx, float** gates, int32_t** perm,
                     int32_t** pos, int32_t** offsets) {
    g_last_error.clear();
    if (int rc = check_dims(d, true)) return rc;
    if (!ws || !topk_idx || !gates || !perm || !pos || !offsets)
        return fail(MOE_ERR_INVALID_ARG, "moe_layer_tables: NULL pointer");
    const LayerWs L = layer_ws(*d, d->T, 1);   // (the tables' offsets do not depend on the threshold)
    char* w = (char*)ws;
    *topk_idx = (int32_t*)(w + L.idx);
    *gates = (float*)(w + L.gates);
    *perm = (int32_t*)(w + L.perm);
    *pos = (int32_t*)(w + L.pos);
    *offsets = (int32_t*)(w + L.offsets);
    return MOE_OK;
}

int moe_quant_rows_f32(const float* v, int rows, int cols, int8_t* q, float* s, cudaStream_t stream) {
    g_last_error.clear();
    if (rows < 0 || cols <= 0) return fail(MOE_ERR_INVALID_ARG, "moe_quant_rows_f32: bad shape");
    if (rows > 0 && (!v || !q || !s)) return fail(MOE_ERR_INVALID_ARG, "moe_quant_rows_f32: NULL pointer");
    cudaError_t e = moe::launch_quant_rows(v, rows, cols, q, s, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_quant_rows_f32 launch");
}

int moe_exp_f32(const float* x, float* y, int64_t n, cudaStream_t stream) {
    g_last_error.clear();
    if (n < 0 || (n > 0 && (!x || !y))) return fail(MOE_ERR_INVALID_ARG, "moe_exp_f32: bad arguments");
    cudaError_t e = moe::launch_exp(x, y, n, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_exp_f32 launch");
}

int moe_swiglu_f32(const float* g, const float* u, float* h, int64_t n, cudaStream_t stream) {
    g_last_error.clear();
    if (n < 0 || (n > 0 && (!g || !u || !h))) return fail(MOE_ERR_INVALID_ARG, "moe_swiglu_f32: bad arguments");
    cudaError_t e = moe::launch_swiglu(g, u, h, n, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_swiglu_f32 launch");
}

// ---- FP8 block-quantised dense projection -----------------------------------

static int check_fp8_dims(int N, int K, const char* who) {
    if (N <= 0 || K <= 0 || N % 128 || K % 128)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: N and K must be positive multiples of 128 (N=%d K=%d)", who, N, K);
    if ((long long)N * K >= (1LL << 40)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s: N*K too large", who);
    return MOE_OK;
}

size_t moe_fp8_packed_bytes(int N, int K) {
    if (N <= 0 || K <= 0 || N % 128 || K % 128) return 0;
    return moe::fp8_packed_bytes(N, K);
}

int moe_fp8_pack_weights(int N, int K, const uint8_t* w_codes, const uint8_t* w_scales, void* packed,
                         cudaStream_t stream) {
    g_last_error.clear();
    if (int rc = check_fp8_dims(N, K, "moe_fp8_pack_weights")) return rc;
    if (!w_codes || !w_scales || !packed) return fail(MOE_ERR_INVALID_ARG, "moe_fp8_pack_weights: NULL pointer");
    if (!aligned(w_codes, 16) || !aligned(packed, 256))
        return fail(MOE_ERR_INVALID_ARG, "moe_fp8_pack_weights: codes need 16-byte, packed 256-byte alignment");
    cudaError_t e = moe::launch_fp8_pack(N, K, w_codes, w_scales, packed, true, nullptr, nullptr, stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_fp8_pack_weights launch");
    int32_t flag = 0;
    e = cudaMemcpyAsync(&flag, (const char*)packed + offsetof(moe::Fp8Header, flag), sizeof(flag),
                        cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_fp8_pack_weights");
    if (flag & MOE_FLAG_BAD_SCALE)
        return fail(MOE_ERR_INVALID_ARG, "moe_fp8_pack_weights: scale byte 0xFF (E8M0 NaN) in the input");
    return MOE_OK;
}

int moe_fp8_unpack_weights(int N, int K, const void* packed, uint8_t* w_codes, uint8_t* w_scales,
                           cudaStream_t stream) {
    g_last_error.clear();
    if (int rc = check_fp8_dims(N, K, "moe_fp8_unpack_weights")) return rc;
    if (!w_codes || !w_scales || !packed) return fail(MOE_ERR_INVALID_ARG, "moe_fp8_unpack_weights: NULL pointer");
    if (!aligned(w_codes, 16) || !aligned(packed, 256))
        return fail(MOE_ERR_INVALID_ARG, "moe_fp8_unpack_weights: codes need 16-byte, packed 256-byte alignment");
    cudaError_t e = moe::launch_fp8_pack(N, K, nullptr, nullptr, const_cast<void*>(packed), false, w_codes, w_scales,
                                         stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_fp8_unpack_weights launch");
}

size_t moe_fp8_workspace_bytes(int T_max, int N, int K) {
    if (T_max < 0 || K <= 0 || K % 128 || N <= 0 || N % 128) return 0;
    return moe::fp8_workspace_bytes(T_max, N, K);
}

int moe_fp8_linear(const void* x_bf16, int T, int N, int K, const void* packed, void* y_bf16, void* ws,
                   size_t ws_bytes, uint8_t* dbg_q, uint8_t* dbg_s, cudaStream_t stream) {
    g_last_error.clear();
    if (int rc = check_fp8_dims(N, K, "moe_fp8_linear")) return rc;
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "moe_fp8_linear: T < 0");
    if ((long long)T * (K > N ? K : N) >= (1LL << 40)) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_fp8_linear: T too large");
    if (!ws || !packed || (T > 0 && (!x_bf16 || !y_bf16)))
        return fail(MOE_ERR_INVALID_ARG, "moe_fp8_linear: NULL pointer");
    if (!aligned(ws, 256) || !aligned(packed, 256) || !aligned(x_bf16, 16) || !aligned(y_bf16, 2) ||
        (dbg_q && !aligned(dbg_q, 16)))
        return fail(MOE_ERR_INVALID_ARG, "moe_fp8_linear: ws/packed need 256-byte, x 16-byte alignment");
    if (ws_bytes < moe::fp8_workspace_bytes(T, N, K))
        return fail(MOE_ERR_INVALID_ARG, "moe_fp8_linear: ws_bytes %zu < %zu", ws_bytes,
                    moe::fp8_workspace_bytes(T, N, K));
    if (T == 0) {
        cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int32_t), stream);
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_fp8_linear memset");
    }
    cudaError_t e = moe::launch_fp8_linear(x_bf16, T, N, K, packed, y_bf16, ws, dbg_q, dbg_s, load_options().wait_ns,
                                           stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_fp8_linear launch");
}

unsigned long long moe_launch_count(void) { return moe::g_launches.load(); }

int moe_set_option(int option, int value) {
    g_last_error.clear();
    if (option == MOE_OPT_TC_MIN_ROWS) {
        if (value < 0) return fail(MOE_ERR_INVALID_ARG, "moe_set_option: TC_MIN_ROWS must be >= 0 (0: automatic)");
        g_tc_min_rows = value;
        return MOE_OK;
    }
    if (option == MOE_OPT_TC_PAIR) {
        if (value != 0 && value != 1) return fail(MOE_ERR_INVALID_ARG, "moe_set_option: TC_PAIR must be 0 or 1");
        g_tc_pair = value;
        return MOE_OK;
    }
    if (option == MOE_OPT_TC_A_TMEM) {
        if (value != 0 && value != 1) return fail(MOE_ERR_INVALID_ARG, "moe_set_option: TC_A_TMEM must be 0 or 1");
        g_tc_a_tmem = value;
        return MOE_OK;
    }
    if (option == MOE_OPT_TC_FORM) {
        if (value < 0 || value > 2) return fail(MOE_ERR_INVALID_ARG, "moe_set_option: TC_FORM must be 0, 1 or 2");
        g_tc_form = value;
        return MOE_OK;
    }
    if (option == MOE_OPT_WAIT_LIMIT_US) {
        if (value < 1 || value > 10000000)
            return fail(MOE_ERR_INVALID_ARG, "moe_set_option: WAIT_LIMIT_US must be in [1, 10^7]");
        g_wait_limit_us = value;
        return MOE_OK;
    }
    if (option == MOE_OPT_TEST_TIMEOUT) {
        if (value != 0 && value != 1) return fail(MOE_ERR_INVALID_ARG, "moe_set_option: TEST_TIMEOUT must be 0 or 1");
        g_test_timeout = value;
        return MOE_OK;
    }
    return fail(MOE_ERR_INVALID_ARG, "moe_set_option: unknown option %d", option);
}

int moe_get_option(int option) {
    if (option == MOE_OPT_TC_MIN_ROWS) return g_tc_min_rows;
    if (option == MOE_OPT_TC_PAIR) return g_tc_pair;
    if (option == MOE_OPT_WAIT_LIMIT_US) return g_wait_limit_us;
    if (option == MOE_OPT_TC_A_TMEM) return g_tc_a_tmem;
    if (option == MOE_OPT_TC_FORM) return g_tc_form;
    if (option == MOE_OPT_TEST_TIMEOUT) return g_test_timeout;
    return -1;
}

int moe_check_device_flag(const void* ws, int32_t* out_flag, cudaStream_t stream) {
    g_last_error.clear();
    if (!ws || !out_flag) return fail(MOE_ERR_INVALID_ARG, "moe_check_device_flag: NULL pointer");
    int32_t f = 0;
    cudaError_t e = cudaMemcpyAsync(&f, ws, sizeof(f), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_check_device_flag");
    *out_flag = f;
    if (f) return fail(MOE_ERR_DEVICE_FLAG, "device error word 0x%x", f);
    return MOE_OK;
}

}  // extern "C"
