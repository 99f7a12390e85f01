// Launch wrappers shared between the kernel files and the C-ABI layer.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstddef>
#include <mutex>

namespace moe {

// Launch set-up computed once per device context: the grid size of a
// persistent kernel and the function attributes it needs (the dynamic
// shared-memory limit is an attribute of the function in the current context).
// get(init) runs init() with the calling thread's device current the first
// time that device -- or a new context on it, after cudaDeviceReset or under a
// caller-created context -- asks, and returns the cached value afterwards.
// init() returns a negative value on failure, which is returned and not cached.
// (The current context is read through the driver entry point that the CUDA
// runtime hands out, so the library does not link against the driver.)
class PerContext {
  public:
    template <class F>
    int get(F init) {
        int dev = 0;
        CUcontext ctx = nullptr;
        const auto get_ctx = ctx_getter();
        if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSlots || !get_ctx ||
            get_ctx(&ctx) != CUDA_SUCCESS)
            return init();
        std::lock_guard<std::mutex> lock(mu_);
        if (ctx_[dev] != ctx || !ctx) {
            const int v = init();
            if (v < 0) return v;
            ctx_[dev] = ctx;
            val_[dev] = v;
        }
        return val_[dev];
    }

  private:
    typedef CUresult (*CtxGetCurrent)(CUcontext*);
    static CtxGetCurrent ctx_getter() {
        static const CtxGetCurrent fn = [] {
            void* p = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess) {
                cudaGetLastError();
                p = nullptr;
            }
            return reinterpret_cast<CtxGetCurrent>(p);
        }();
        return fn;
    }
    static constexpr int kSlots = 64;
    std::mutex mu_;
    CUcontext ctx_[kSlots] = {};
    int val_[kSlots] = {};
};

// Unit of the streaming grouped GEMM: kGemvTileRows weight rows by up to
// kGemvGroup token rows (shared by it and the planner).
constexpr int kGemvTileRows = 64;
constexpr int kGemvGroup = 4;   // 6 and 8 measured slower on decode_T8 and decode_T64
constexpr int kGemvSmallGroup = 2;       // token rows per unit for calls with T <= kGemvSmallGroupMaxT
constexpr int kGemvSmallGroupMaxT = 16;
// Tile of the tensor-core grouped GEMM: 128 weight rows (the MMA's M) by up to
// 128 sorted token rows (its N); shared by the planner and the kernel.
constexpr int kMaxExperts = 1024;   // the API's limit on E
constexpr int kTcWeightTile = 128;
constexpr int kTcTokenTile = 128;
// Weight rows per tile of the token-major form (tc_gemm_tn.cu): two packed
// 128-row chunks.
constexpr int kTcTnWeightTile = 256;
// Token tile of the tensor-core GEMM's decode configuration (calls with at
// most kTcDecodeMaxT tokens, so at most that many rows per expert).
constexpr int kTcDecodeTokenTile = 32;
constexpr int kTcDecodeMaxT = 64;

// Number of kernels this library has launched in the process (diagnostics).
void count_launches(int n);

cudaError_t launch_plan_rows(const int32_t* offsets, const int32_t* topk_idx, const int32_t* perm, int E, int P,
                             int I, int H, int tc_min, int tc_tile1, int tc_tile2, int tc_wtile1, int tc_wtile2,
                             int group, int32_t* unit_off1, int32_t* unit_off2, int32_t* tile_off1,
                             int32_t* tile_off2, int32_t* plane_off, int32_t* stream_off, int32_t* expert_tc,
                             int32_t* plane_row, double* gacc, double* yacc, int32_t* flag, cudaStream_t st);

// Launch with programmatic dependent launch allowed: the kernel may be
// scheduled before the preceding kernel in the stream completes.  Every kernel
// launched this way starts with pdl_begin() (moe_common.cuh), which waits for
// that kernel (and so, transitively, for every earlier one) before touching
// memory.  This hides the launch gap between the layer's short kernels.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct PackedLayout {
    size_t header, w1, w1_expert_bytes, w2, w2_expert_bytes, total;
};
PackedLayout packed_layout(int H, int I, int E);

cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* gates,
                         cudaStream_t st);
cudaError_t launch_router_logits(const void* x, const float* wr, const float* bias, int T, int H, int E,
                                 float* logits, cudaStream_t st);

// Route, sort, x quant and plan of a layer call in one launch (front.cu), for
// calls with no tensor-core expert and at most kFrontMaxPairs pairs.
constexpr int kFrontMaxPairs = 1024;
cudaError_t launch_layer_front(const float* logits, const void* x, const void* packed, int T, int H, int I,
                               int E, int k, int group, int32_t* topk_idx, float* gates, int32_t* perm, int32_t* pos,
                               int32_t* offsets, int32_t* unit_off1, int32_t* unit_off2, int32_t* plane_row, int8_t* xq, float* sx, int32_t* xinit, int8_t* dbg_xq,
                               float* dbg_sx, double* gacc, double* yacc, int32_t* flag, cudaStream_t st);

size_t sort_workspace_bytes(int T_max, int k, int E);
cudaError_t launch_sort(const int32_t* topk_idx, int T, int k, int E, int32_t* perm, int32_t* pos,
                        int32_t* offsets, void* ws, cudaStream_t st);

int sort_static_fits(int T, int k, int E);
cudaError_t launch_sort_static(const int32_t* topk_idx, int T, int k, int E, int32_t* perm,
                               int32_t* pos, int32_t* offsets, cudaStream_t st);

cudaError_t launch_pack(int H, int I, int E, const uint8_t* w1c, const uint8_t* w1s,
                        const uint8_t* w2c, const uint8_t* w2s, void* packed, bool forward,
                        uint8_t* out_w1c, uint8_t* out_w1s, uint8_t* out_w2c, uint8_t* out_w2s,
                        cudaStream_t st);
const int32_t* packed_flag_ptr(const void* packed);


cudaError_t launch_xquant(const void* x, int T, int H, int8_t* xq, float* sx, int32_t* xinit,
                          uint8_t* tplanes, int8_t* dbg_xq, float* dbg_sx, const void* packed, int I, int E,
                          int32_t* flag, cudaStream_t st);
cudaError_t launch_hquant(const double* gacc, float* hbuf, const float* sx, const int32_t* perm,
                          const int32_t* plane_row, int plane_rows, int stream_rows, uint8_t* planes, int P, int k,
                          int I, int8_t* hq, float* sh, int32_t* hinit, int8_t* dbg_hq, float* dbg_sh, int32_t* flag,
                          cudaStream_t st);

cudaError_t launch_exp(const float* x, float* y, int64_t n, cudaStream_t st);
cudaError_t launch_swiglu(const float* g, const float* u, float* h, int64_t n, cudaStream_t st);
cudaError_t launch_quant_rows(const float* v, int rows, int cols, int8_t* q, float* s,
                              cudaStream_t st);


cudaError_t launch_gemv(const uint8_t* w, size_t expert_bytes, int K, int N, const int8_t* act,
                        const int32_t* act_init, const int32_t* perm, int k_div,
                        const int32_t* offsets, const int32_t* unit_off, const int32_t* stream_off, int E,
                        double* out, const int32_t* flag, int gate_up_half, int P, int group, bool pre_wait,
                        cudaStream_t st);

size_t tc_smem_bytes();
// Digit planes, per 128-input stage g and group of 8 plane rows, hold
// [plane 0..2][32-input chunk 0..3][8 rows][16 bytes] (1536 bytes); plane rows
// are the sorted rows of tensor-core experts, each expert padded to 16 rows.
constexpr int kPlaneGroupBytes = 1536;
__host__ __device__ inline size_t plane_bytes(int K, int plane_rows) {
    return (size_t)(K / 128) * (plane_rows / 8) * kPlaneGroupBytes;
}
cudaError_t launch_planes(const uint8_t* tplanes, int K, const int32_t* perm, int k_div, int rows,
                          const int32_t* plane_row, int plane_rows, uint8_t* planes, int32_t* flag,
                          cudaStream_t st);
cudaError_t launch_tc_gemm(const uint8_t* w, size_t expert_bytes, int K, int N, int gate_up_half,
                           const uint8_t* planes, int plane_rows, const int32_t* plane_off, int P,
                           const int32_t* offsets, const int32_t* tile_off, int E, int32_t* flag,
                           const float* row_scale, const int32_t* perm, int k_div, float* out, int token_tile,
                           bool pair, bool a_tmem, uint64_t wait_ns, int withhold, cudaStream_t st);

// expert_tc == NULL (the fused decode front): every row is a streaming row at
// its sorted row; otherwise the kind and the compact streaming row come from
// expert_tc / offsets / stream_off of the planner.
// Token-major form (tc_gemm_tn.cu): 128 token rows x 256 weight rows per tile,
// tile_off counting 256-row weight blocks; the same arguments otherwise.
cudaError_t launch_tc_gemm_tn(const uint8_t* w, size_t expert_bytes, int K, int N, int gate_up_half,
                              const uint8_t* planes, int plane_rows, const int32_t* plane_off, int P,
                              const int32_t* offsets, const int32_t* tile_off, int E, int32_t* flag,
                              const float* row_scale, const int32_t* perm, int k_div, float* out, uint64_t wait_ns,
                              int withhold, cudaStream_t st);

cudaError_t launch_combine(const double* yacc, const float* yf, const int32_t* expert_tc, const int32_t* offsets,
                           const int32_t* stream_off, const int32_t* topk_idx, int E, int stream_rows,
                           const float* sh, const float* gates, const int32_t* pos, int T, int k, int H, void* y,
                           int32_t* flag, cudaStream_t st);

// ---- FP8 block-quantised dense projection (fp8_gemm.cu) ----
constexpr int kFp8ChunkBytes = 512 + 128 * 128;   // scale atom + 128 x 128 E4M3 codes
constexpr size_t kFp8HeaderBytes = 256;
constexpr uint32_t kFp8Magic = 0x57385046u;      // "FP8W"
struct Fp8Header {
    uint32_t magic, N, K, reserved;
    int32_t flag;  // device error word of the packing
};
size_t fp8_packed_bytes(int N, int K);
// Calls of at most kFp8SplitMaxT tokens split each tile's K range over up to
// kFp8MaxSplits CTAs (fp32 partials in the workspace).
constexpr int kFp8SplitMaxT = 64;
constexpr int kFp8MaxSplits = 8;
size_t fp8_workspace_bytes(int T, int N, int K);
cudaError_t launch_fp8_pack(int N, int K, const uint8_t* wq, const uint8_t* ws, void* packed, bool fwd,
                            uint8_t* out_wq, uint8_t* out_ws, cudaStream_t st);
cudaError_t launch_fp8_linear(const void* x, int T, int N, int K, const void* packed, void* y, void* ws,
                              uint8_t* dbg_q, uint8_t* dbg_s, uint64_t wait_ns, cudaStream_t st);

}  // namespace moe
