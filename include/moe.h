/*
 * moe.h -- C ABI of the B200 (sm_100a) routed FP4 mixture-of-experts layer.
 *
 * The layer is the routed mixture-of-experts block of DeepSeek-V4-Flash-style
 * inference.  Sources:
 *   [A] "DeepSeek-V4-Flash on AMD gfx90a: Correctness Recovery and Inference
 *       Performance Engineering", abstract: FP4 routed mixture-of-experts,
 *       packed FP4 weights, INT8 activation quantisation, expert sorting, the
 *       W2 expert projection whose load-time layout had to be repaired, and
 *       fixed-token / hash-based correctness checks.
 *   [B] "DeepSeek V4 Flash on 8x R9600D" (blog post), model facts paragraph:
 *       256 routed experts, 6 active per token, FP4 expert weights.
 * The pages name these steps without formulas; the formulas stated below are
 * the readings this library implements (and its CPU oracle checks).
 *
 * Conventions for every call
 *   - Tensor pointers are DEVICE pointers owned by the caller, unless a comment
 *     says otherwise.  The library never allocates or frees device memory.
 *   - Calls are asynchronous on `stream` and never synchronise the host, except
 *     moe_pack_weights and moe_check_device_flag (load-time / test calls that
 *     say so).  moe_route, moe_sort, moe_forward and moe_layer_forward can be
 *     captured in a CUDA graph.
 *   - Kernels are launched with programmatic dependent launch: a kernel may be
 *     scheduled while the previous kernel on `stream` finishes, but it waits for
 *     that kernel to complete before it touches memory, so stream order holds
 *     for the caller's own work before and after every call.
 *   - Return value: MOE_OK, or a negative moe_status.  Host-side argument
 *     checks fail before anything is launched; moe_last_error() returns the
 *     message of the calling thread's last failure.
 *   - Errors found on the device (bad expert id, NaN scale byte, packed-header
 *     mismatch) never trap: kernels OR a bit into the int32 at offset 0 of the
 *     workspace, which moe_check_device_flag() reads.
 *   - Row-major layouts throughout.  "Sorted order" means the order of moe_sort's
 *     permutation: row i holds pair perm[i].
 *   - Shapes: H % 128 == 0, I % 128 == 0, 1 <= k <= min(E, 16), E <= 1024,
 *     T >= 0, T * k < 2^31.
 */
#ifndef FP4_ROUTED_MOE_H
#define FP4_ROUTED_MOE_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,      /* NULL pointer, bad size, misaligned buffer, NaN scale */
    MOE_ERR_UNSUPPORTED_SHAPE = -2,/* dims outside the supported set */
    MOE_ERR_CUDA = -3,             /* a CUDA runtime call or launch failed */
    MOE_ERR_LAYOUT_MISMATCH = -4,  /* packed weights were built for other dims */
    MOE_ERR_TIMEOUT = -5,          /* a bounded device wait gave up */
    MOE_ERR_DEVICE_FLAG = -6       /* moe_check_device_flag found a raised bit */
} moe_status;

/* Bits of the device error word (see moe_check_device_flag). */
#define MOE_FLAG_BAD_EXPERT 1
#define MOE_FLAG_BAD_SCALE 2
#define MOE_FLAG_LAYOUT 4
#define MOE_FLAG_TIMEOUT 8
#define MOE_FLAG_BOUNDS 16

/* T tokens of hidden size H; E routed experts with intermediate size I; k
 * experts per token ([B]: E = 256, k = 6). */
typedef struct {
    int T, H, I, E, k;
} moe_dims;

/* Optional dumps of the INT8 activations for bit-exact checks, and optional
 * timing events; any member may be NULL.  xq [T,H] int8 and sx [T] fp32 in
 * token order; hq [T*k, I] int8 and sh [T*k] fp32 in sorted order.
 * events[0..3], when set, are recorded on the call's stream right before and
 * after the W1 GEMM and right before and after the W2 GEMM (caller-created
 * events; recording them adds no synchronisation). */
typedef struct {
    int8_t *xq;
    float *sx;
    int8_t *hq;
    float *sh;
    cudaEvent_t events[4];
} moe_debug;

/* Message of the calling thread's last failed call (empty if none); copies at
 * most n bytes including the terminating NUL.  Returns the full length. */
size_t moe_last_error(char *buf, size_t n);

/* ---------------------------------------------------------------------------
 * Weights ([A]: packed FP4 expert weights; the W2 layout bug and its repair at
 * load time).
 *
 * Canonical MXFP4 input (host-visible definition, device memory):
 *   w1_codes  [E, 2I, H/2] uint8   W1 rows [0,I) gate, [I,2I) up; byte j of a
 *                                  row holds element 2j in its low nibble and
 *                                  2j+1 in its high nibble; nibble = E2M1 code
 *   w1_scales [E, 2I, H/32] uint8  UE8M0: element k of row n is
 *                                  e2m1(code) * 2^(scale[n, k/32] - 127)
 *   w2_codes  [E, H, I/2], w2_scales [E, H, I/32]: the same for W2.
 * Scale byte 0xFF (NaN) is rejected.
 * ------------------------------------------------------------------------- */

/* Size in bytes of the device layout built by moe_pack_weights. */
size_t moe_packed_bytes(const moe_dims *d);

/* Canonical -> device layout.  `packed` must hold moe_packed_bytes(d) bytes,
 * 256-byte aligned.  Load-time call: it SYNCHRONISES `stream` and returns
 * MOE_ERR_INVALID_ARG if any scale byte is 0xFF (the output is then unusable). */
int moe_pack_weights(const moe_dims *d, const uint8_t *w1_codes, const uint8_t *w1_scales,
                     const uint8_t *w2_codes, const uint8_t *w2_scales, void *packed,
                     cudaStream_t stream);

/* Device layout -> canonical (the exact inverse of moe_pack_weights).  The
 * round trip must reproduce the canonical bytes exactly; callers compare them
 * once at load time, which catches any layout permutation.  Asynchronous. */
int moe_unpack_weights(const moe_dims *d, const void *packed, uint8_t *w1_codes,
                       uint8_t *w1_scales, uint8_t *w2_codes, uint8_t *w2_scales,
                       cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Router projection ([B]: one logit per routed expert), in front of routing:
 *   logits[t, e] = sum_h x[t, h] * w_router[e, h] (+ bias[e])
 * x [T, H] bf16 (16-byte aligned), w_router [E, H] fp32 (16-byte aligned),
 * bias [E] fp32 or NULL, logits [T, E] fp32; all device pointers owned by the
 * caller.  fp32 fused multiply-adds in ascending h: |logits - S| <=
 * gamma_(H+1) * sum_h |x w| plus one rounding of the bias addition, where S is
 * the exact value and gamma_n = n u / (1 - n u), u = 2^-24.  H % 32 == 0,
 * 1 <= E <= 1024.  Asynchronous, graph-capturable; MOE_ERR_INVALID_ARG on NULL
 * or misaligned pointers, MOE_ERR_UNSUPPORTED_SHAPE on other shapes.
 * ------------------------------------------------------------------------- */
int moe_router_logits(const void *x_bf16, const float *w_router, const float *bias, int T, int H,
                      int E, float *logits, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Routing ([B]: each token picks k of E routed experts).
 * logits [T, E] fp32 -> topk_idx [T, k] int32, gates [T, k] fp32.
 * topk_idx[t] lists the k largest logits in descending order, equal logits
 * going to the lower expert id and NaN ranking below every number.
 * gates[t, j] = exp(l_j - l_0) / sum_{j'<k} exp(l_j' - l_0): the softmax over
 * all E experts renormalised over the chosen k (the full denominator cancels);
 * no routed scaling factor.  exp is the library's fp32 exp.
 * ------------------------------------------------------------------------- */
int moe_route(const float *logits, int T, int E, int k, int32_t *topk_idx, float *gates,
              cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Expert sorting ([A]: expert sorting before the expert GEMMs).
 * Stable counting sort of the P = T*k token-expert pairs (pair id p = t*k + j)
 * by expert id topk_idx[p]:
 *   offsets [E+1] int32: offsets[e] = number of pairs with expert < e;
 *   perm    [P] int32:   pair ids grouped by expert, ascending inside a group;
 *   pos     [P] int32:   inverse permutation, pos[perm[i]] = i.
 * ws: moe_sort_workspace_bytes(T, k, E) bytes, 256-byte aligned, any contents.
 * An expert id outside [0, E) raises MOE_FLAG_BAD_EXPERT in ws; such pairs are
 * left out of the sort: perm/pos are then incomplete and offsets[E], the
 * number of pairs sorted, is below T*k.
 * ------------------------------------------------------------------------- */
size_t moe_sort_workspace_bytes(int T_max, int k, int E);
int moe_sort(const int32_t *topk_idx, int T, int k, int E, int32_t *perm, int32_t *pos,
             int32_t *offsets, void *ws, size_t ws_bytes, cudaStream_t stream);

/* moe_sort without a workspace argument.  The paper has no counterpart: this
 * entry point exists for callers that are handed only input and output
 * buffers -- for example code embedded in a host framework that owns all
 * device memory and offers no way to request a scratch buffer -- and so cannot
 * call cudaMalloc or size a workspace themselves.  Same arguments (minus ws)
 * and same results as moe_sort; nothing is allocated.
 *   - Scratch is a fixed 256 KB array inside the library (held on every GPU
 *     that loads it, until process exit): T*k <= 65536 pairs and E <= 1024;
 *     larger calls return MOE_ERR_UNSUPPORTED_SHAPE (use moe_sort).
 *   - Every call looks up that array's device address in the calling
 *     thread's current context (cudaGetSymbolAddress; the address belongs to
 *     the library's module in that context, so it is not cached).  The first
 *     call in a context may load the module: make it before any stream
 *     capture.
 *   - All calls share the array: calls that overlap on a GPU race.  Each call
 *     clears and rewrites what it reads.
 *   - Expert ids outside [0, E) are skipped as in moe_sort.  The caller sees
 *     it in the outputs, without any extra read: offsets[E] is the number of
 *     pairs sorted, so offsets[E] < T*k means that T*k - offsets[E] pairs had
 *     a bad id (and perm/pos are incomplete). */
int moe_sort_static(const int32_t *topk_idx, int T, int k, int E, int32_t *perm, int32_t *pos,
                    int32_t *offsets, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The expert computation ([A]: INT8 activation quantisation, packed FP4
 * expert GEMMs W1 and W2; routed mixture combine).
 *   xq, sx  = per-token symmetric INT8 of x: sx = fp32(max|x_t| / 127),
 *             xq = clamp(rne(fp32(x / sx)), -127, 127)  (0 when the row is 0)
 *   G[i, n] = fp32( fp64(sx[t]) * sum_k xq[t,k] * w1[e, n, k] ),  n < 2I
 *   h[i, n] = fp32( fp32(g / fp32(1 + exp(-g))) * u ), g = G[i,n], u = G[i,I+n]
 *   hq, sh  = per-row symmetric INT8 of h (same rule as x)
 *   Y[i, n] = fp32( fp64(sh[i]) * sum_j hq[i,j] * w2[e, n, j] ),  n < H
 *   y[t, n] = bf16( sum_{j<k} gates[t,j] * Y[pos[t*k+j], n] )   (fp32 sum, slot order)
 * for every sorted row i = pos[t*k+j] with e = topk_idx[t*k+j].  The sums over
 * k and j are exact (integer-valued products in units of half the row's
 * smallest weight scale): in the streaming GEMM (fp64 block sums) while a row's
 * scale bytes span less than about 28 binades, in the tensor-core GEMM (fp32
 * accumulators) while every partial sum stays below 2^24 of those units.
 * x [T, H] bf16, y [T, H] bf16; the other pointers as produced by moe_route /
 * moe_sort; packed from moe_pack_weights with the same H, I, E.
 * ws: moe_workspace_bytes(d, T_max) bytes, 256-byte aligned, T <= T_max; its
 * first int32 is the device error word and is cleared by this call.
 * dbg: NULL in the hot path.  T == 0 is a no-op.
 * ------------------------------------------------------------------------- */
size_t moe_workspace_bytes(const moe_dims *d, int T_max);
int moe_forward(const moe_dims *d, const void *x_bf16, const int32_t *topk_idx,
                const float *gates, const int32_t *perm, const int32_t *pos,
                const int32_t *offsets, const void *packed, void *y_bf16, void *ws,
                size_t ws_bytes, const moe_debug *dbg, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The whole layer in one call: moe_route, moe_sort and moe_forward on one
 * stream, from router logits [T, E] fp32 and x [T, H] bf16 to y [T, H] bf16.
 * ws: moe_layer_workspace_bytes(d, T_max) bytes, 256-byte aligned, T <= T_max;
 * it holds the forward workspace (device error word first), the routing and
 * sort outputs and the sort scratch.  Asynchronous, graph-capturable.
 * Decode-size calls (0 < T < MOE_OPT_TC_MIN_ROWS and T * k <= 1024, so that
 * every expert takes the streaming GEMM) run route, sort, x quant and the
 * work plan as one fused launch; the results are the same as those of the
 * separate calls (the same device code runs in both).
 * ------------------------------------------------------------------------- */
size_t moe_layer_workspace_bytes(const moe_dims *d, int T_max);
int moe_layer_forward(const moe_dims *d, const float *logits, const void *x_bf16,
                      const void *packed, void *y_bf16, void *ws, size_t ws_bytes,
                      const moe_debug *dbg, cudaStream_t stream);

/* The router projection followed by the whole layer: logits = x W_router^T
 * (+ bias), as moe_router_logits computes them, then moe_layer_forward on
 * those logits -- from x [T, H] bf16, w_router [E, H] fp32 and bias [E] fp32
 * (or NULL) to y [T, H] bf16.  ws: moe_layer_router_workspace_bytes(d, T_max)
 * bytes, 256-byte aligned, T <= T_max: the layer workspace (error word first;
 * moe_layer_tables works on it) followed by the logits.  The results equal
 * those of moe_router_logits followed by moe_layer_forward.  Asynchronous,
 * graph-capturable; errors as for those two calls. */
size_t moe_layer_router_workspace_bytes(const moe_dims *d, int T_max);
int moe_layer_forward_with_router(const moe_dims *d, const void *x_bf16, const float *w_router,
                                  const float *bias, const void *packed, void *y_bf16, void *ws,
                                  size_t ws_bytes, const moe_debug *dbg, cudaStream_t stream);

/* Device pointers to the routing tables moe_layer_forward leaves in its
 * workspace `ws` for dims d (d->T = the call's T): topk_idx [T, k] and gates
 * [T, k] as moe_route writes them, perm [T*k], pos [T*k] and offsets [E + 1]
 * as moe_sort writes them.  Pure pointer arithmetic (nothing is launched or
 * read); the tables are valid once that call has completed on its stream and
 * until the next call that uses ws.  MOE_ERR_INVALID_ARG on NULL pointers. */
int moe_layer_tables(const moe_dims *d, void *ws, int32_t **topk_idx, float **gates,
                     int32_t **perm, int32_t **pos, int32_t **offsets);

/* Stage entry point: per-row symmetric INT8 quantisation of fp32 rows
 * v [rows, cols] -> q [rows, cols] int8, s [rows] fp32 (rule as for x above). */
int moe_quant_rows_f32(const float *v, int rows, int cols, int8_t *q, float *s,
                       cudaStream_t stream);

/* Stage entry points of the layer's fp32 exp and SwiGLU (the functions used
 * inside moe_route and moe_forward), for bit-exact checks:
 *   y[i] = exp(x[i]) (Cody-Waite reduction, degree-7 Taylor polynomial,
 *          fused multiply-adds; +inf above 88.8, 0 below -104);
 *   h[i] = fp32( fp32(g[i] / fp32(1 + exp(-g[i]))) * u[i] ).
 * fp32 device arrays of n elements. */
int moe_exp_f32(const float *x, float *y, int64_t n, cudaStream_t stream);
int moe_swiglu_f32(const float *g, const float *u, float *h, int64_t n, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * FP8 block-quantised dense projection ([A]: FP8 dense projections; [B]:
 * "FP8 block quantization").  Readings: OCP E4M3 codes; one UE8M0 scale
 * (value 2^(byte - 127)) per 128 x 128 weight block and per token x
 * 128-input activation block;
 *   xq, sx  per token and 128-input block of x: sx = the smallest power of two
 *           2^e with max|x| <= 448 * 2^e (byte e + 127, 0 for an all-zero
 *           block), xq = E4M3 codes of x / 2^e, round to nearest even;
 *   y[t, n] = bf16( sum_k xq[t,k] 2^(sx[t,k/128]-127) * wq[n,k] 2^(sw[n/128,k/128]-127) )
 * accumulated in fp32 by the tensor cores (tcgen05 kind::mxf8f6f4 with block
 * scaling), rounded once to bf16.
 * Weights, canonical (device memory): w_codes [N, K] uint8 E4M3 codes,
 * w_scales [N/128, K/128] uint8 UE8M0 bytes; 0xFF (NaN) is rejected.
 * N % 128 == 0, K % 128 == 0.
 * ------------------------------------------------------------------------- */

/* Size of the device layout built by moe_fp8_pack_weights (0 for bad dims). */
size_t moe_fp8_packed_bytes(int N, int K);

/* Canonical -> device layout (256-byte header, then 128 x 128 chunks).
 * `packed`: moe_fp8_packed_bytes bytes, 256-byte aligned; w_codes 16-byte
 * aligned.  Load-time call: SYNCHRONISES `stream`; MOE_ERR_INVALID_ARG on a
 * scale byte 0xFF. */
int moe_fp8_pack_weights(int N, int K, const uint8_t *w_codes, const uint8_t *w_scales, void *packed,
                         cudaStream_t stream);

/* Device layout -> canonical, the exact inverse (a round-trip check at load
 * time catches any layout permutation).  Asynchronous. */
int moe_fp8_unpack_weights(int N, int K, const void *packed, uint8_t *w_codes, uint8_t *w_scales,
                           cudaStream_t stream);

/* Workspace of moe_fp8_linear for up to T_max tokens, N outputs and K inputs
 * (error word first; the quantised activations in the GEMM's tile order; for
 * calls of at most 64 tokens, whose tiles' K ranges are split over several
 * CTAs, the fp32 partial sums).  0 for invalid dims. */
size_t moe_fp8_workspace_bytes(int T_max, int N, int K);

/* y [T, N] bf16 = the projection of x [T, K] bf16 (16-byte aligned) by the
 * packed weights.  ws: moe_fp8_workspace_bytes(T_max, N, K) bytes, 256-byte
 * aligned, T <= T_max; its first int32 is the device error word (cleared by
 * this call; MOE_FLAG_LAYOUT when `packed` was built for other N, K; the GEMM
 * then leaves y untouched; MOE_FLAG_TIMEOUT as in moe_forward).  dbg_q
 * [T, K] (16-byte aligned) and dbg_s [T, K/128], when not NULL, receive the
 * E4M3 codes and UE8M0 bytes of x.  Asynchronous, graph-capturable. */
int moe_fp8_linear(const void *x_bf16, int T, int N, int K, const void *packed, void *y_bf16, void *ws,
                   size_t ws_bytes, uint8_t *dbg_q, uint8_t *dbg_s, cudaStream_t stream);

/* Process-wide options.  Each call reads them once when it starts, so a call
 * sees one consistent set; a change made while calls are being enqueued on
 * other host threads applies from the next call that starts after it.
 *   MOE_OPT_TC_MIN_ROWS: experts with at least this many token rows in a call
 *   run on the tensor-core grouped GEMMs (tcgen05, forms: MOE_OPT_TC_FORM);
 *   experts with fewer rows run on the CUDA-core streaming GEMM.  Both paths give the
 *   same results inside the exactness domains stated at moe_forward.
 *   0 (the default) is automatic: calls of fewer than 32 tokens run every
 *   expert on the streaming GEMM (and moe_layer_forward fuses their route,
 *   sort, x quant and plan into one launch), larger calls use a threshold of
 *   2.  A value >= 1 is used as it is.  The forward workspace depends on this
 *   option: size it after setting the option.
 *   MOE_OPT_TC_FORM: the forms of the tensor-core GEMMs.  0 (default): W1
 *   token-major (128 token rows as the MMA's M, two 128-row weight chunks as
 *   N: the activation operand is staged once for 256 weight rows), W2
 *   weight-major (128 weight rows as M, token rows as N: its fp32 output rows
 *   are stored in whole lines; 128-row token tiles, or 32-row ones in calls of
 *   at most 64 tokens); 1: both weight-major; 2: both token-major.  Same
 *   results.
 *   MOE_OPT_TC_PAIR: 1 runs both tensor-core GEMMs weight-major in SM pairs
 *   (clusters of two CTAs, tcgen05 cta_group::2, M = 256) where the weight
 *   rows allow it (a multiple of 256); 0 one CTA per SM.  Same results.
 *   MOE_OPT_TC_A_TMEM: 1 runs both tensor-core GEMMs weight-major with each
 *   pipeline stage's weight chunk staged in tensor memory once (tcgen05.cp)
 *   and the six digit-plane MMAs of the stage reading A from there, so shared
 *   memory feeds only the activation operand; 0 reads both operands from
 *   shared memory.  One CTA per SM (it takes precedence over
 *   MOE_OPT_TC_PAIR).  Same results.
 *   MOE_OPT_WAIT_LIMIT_US: limit, in microseconds, of every bounded wait inside
 *   the tensor-core GEMM (a pipeline stage normally lands in a few
 *   microseconds).  A wait that runs out raises MOE_FLAG_TIMEOUT in the call's
 *   error word; the kernel still waits (again bounded) for its own copies and
 *   MMAs, frees its tensor memory and returns, and the call's results are
 *   invalid.  Default 1000000 (one second); range [1, 10^7].
 *   MOE_OPT_TEST_TIMEOUT: 1 arms a test of that path: the next call that runs
 *   the tensor-core W1 GEMM has its first CTA's first pipeline stage withheld
 *   (neither copied nor signalled), so the MMA waiting for it runs out of
 *   time.  The arming is consumed by that call; 0 disarms.  For tests only.
 * moe_set_option returns MOE_OK or MOE_ERR_INVALID_ARG; moe_get_option returns
 * the current value (-1 for an unknown option). */
#define MOE_OPT_TC_MIN_ROWS 1
#define MOE_OPT_TC_PAIR 2
#define MOE_OPT_WAIT_LIMIT_US 3
#define MOE_OPT_TEST_TIMEOUT 4
#define MOE_OPT_TC_A_TMEM 5
#define MOE_OPT_TC_FORM 6
int moe_set_option(int option, int value);
int moe_get_option(int option);

/* Number of CUDA kernels this library has launched in the calling process
 * (a diagnostic counter; memsets and event records are not counted). */
unsigned long long moe_launch_count(void);

/* Reads the device error word at the start of `ws` into *out_flag (host
 * pointer).  SYNCHRONISES `stream`: tests and diagnostics only.  Returns
 * MOE_ERR_DEVICE_FLAG when a bit is set, else MOE_OK. */
int moe_check_device_flag(const void *ws, int32_t *out_flag, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* FP4_ROUTED_MOE_H */
