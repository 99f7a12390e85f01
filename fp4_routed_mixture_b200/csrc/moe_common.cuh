// Shared device helpers of the routed FP4 MoE library (sm_100a).
//
// Exactness-sensitive arithmetic uses explicit round-to-nearest intrinsics
// (__fmul_rn, __fadd_rn, __fmaf_rn, __fdiv_rn, __dmul_rn) so that no
// contraction or approximation changes a rounding.  The library is built
// without --use_fast_math.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Bits of the device-side error word (first int32 of a workspace).
enum : int32_t {
    FLAG_BAD_EXPERT = 1,   // an expert id outside [0, E) reached moe_sort
    FLAG_BAD_SCALE = 2,    // a UE8M0 scale byte 0xFF (NaN) reached moe_pack_weights
    FLAG_LAYOUT = 4,       // the packed weight header does not match the dims
    FLAG_TIMEOUT = 8,      // a bounded device wait gave up
    FLAG_BOUNDS = 16,      // an index check failed inside a kernel
};

__device__ __forceinline__ void raise_flag(int32_t* flag, int32_t bit) {
    if (flag) atomicOr(flag, bit);
}

// An index read from a caller-provided table (perm, pos, topk_idx): values
// outside [0, n) raise FLAG_BOUNDS and are replaced by 0, so a bad table can
// give wrong results but never an out-of-bounds access.
__device__ __forceinline__ int checked_index(int v, int n, int32_t* flag) {
    if ((unsigned)v < (unsigned)n) return v;
    raise_flag(flag, FLAG_BOUNDS);
    return 0;
}

// ---- The layer's fp32 exp ---------------------------------------------------
// Cody-Waite argument reduction (ln 2 split into a short exact high part and a
// low part) followed by a Taylor polynomial; written from the mathematics.
// Specification (the CPU reference implements the same one separately):
//   NaN -> NaN; x > 88.8 -> +inf; x < -104 -> 0;
//   n = rint(fp32(x * log2e)); r = fma(-n, ln2_hi, x); r = fma(-n, ln2_lo, r);
//   p = Horner over 1/j!, j = 7..0, with fused multiply-adds;
//   result = p * 2^n, split into two exact-or-final multiplies at the ends of
//   the exponent range.
// log2e = fp32(1/ln 2); ln2_hi = ln 2 truncated to 12 significant bits;
// ln2_lo = fp32(ln 2 - ln2_hi); the Taylor coefficients are fp32(1/j!).
__device__ __forceinline__ float pow2i(int n) { return __int_as_float((n + 127) << 23); }

__device__ __forceinline__ float layer_exp(float x) {
    if (x != x) return x;
    if (x > 88.8f) return __int_as_float(0x7f800000);
    if (x < -104.0f) return 0.0f;
    const float nf = rintf(__fmul_rn(x, 1.44269502162933349609375f));
    float r = __fmaf_rn(-nf, 0.693115234375f, x);
    r = __fmaf_rn(-nf, 3.19461832987144589424133e-05f, r);
    float p = 0.00019841270113829523324966431f;            // 1/7!
    p = __fmaf_rn(p, r, 0.0013888889225199818611145020f);  // 1/6!
    p = __fmaf_rn(p, r, 0.0083333337679505348205566406f);  // 1/5!
    p = __fmaf_rn(p, r, 0.041666667908430099487304688f);   // 1/4!
    p = __fmaf_rn(p, r, 0.16666667163372039794921875f);    // 1/3!
    p = __fmaf_rn(p, r, 0.5f);                             // 1/2!
    p = __fmaf_rn(p, r, 1.0f);                             // 1/1!
    p = __fmaf_rn(p, r, 1.0f);                             // 1/0!
    const int n = (int)nf;
    if (n > 126) return __fmul_rn(__fmul_rn(p, pow2i(n - 1)), 2.0f);
    if (n < -125) return __fmul_rn(__fmul_rn(p, pow2i(n + 100)), pow2i(-100));
    return __fmul_rn(p, pow2i(n));
}

// SwiGLU: h = fp32( fp32(g / fp32(1 + exp(-g))) * u ), no clamp.
__device__ __forceinline__ float swiglu(float g, float u) {
    const float d = __fadd_rn(1.0f, layer_exp(-g));
    return __fmul_rn(__fdiv_rn(g, d), u);
}

// Symmetric INT8 code of v for a row with absolute maximum a and scale
// s = fp32(a / 127): clamp(round-half-even(fp32(v / s)), -127, 127); 0 when a == 0.
__device__ __forceinline__ float quant_scale(float amax) { return __fdiv_rn(amax, 127.0f); }

__device__ __forceinline__ int quant_code(float v, float amax, float s) {
    if (amax == 0.0f) return 0;
    float r = rintf(__fdiv_rn(v, s));
    r = fminf(127.0f, fmaxf(-127.0f, r));
    return (int)r;
}

// Header at the start of a packed weight buffer (written by moe_pack_weights).
struct PackHeader {
    uint32_t magic, version, H, I, E, reserved0;
    uint64_t w1_off, w2_off;
    int32_t flag;  // device error word of moe_pack_weights
};
constexpr uint32_t kPackMagic = 0x34454F4Du;  // "MOE4"
constexpr uint32_t kPackVersion = 3;

// True when the packed buffer was built for these dims (a mismatch raises
// FLAG_LAYOUT and keeps the GEMMs out of the buffer).
__device__ __forceinline__ bool packed_header_ok(const void* packed, int H, int I, int E) {
    const PackHeader* h = reinterpret_cast<const PackHeader*>(packed);
    return h->magic == kPackMagic && h->version == kPackVersion && (int)h->H == H && (int)h->I == I &&
           (int)h->E == E;
}

// First statement of every kernel launched with launch_pdl: wait until the
// preceding kernel in the stream has completed and its writes are visible,
// then allow the next kernel to be scheduled (it waits in turn, so at most two
// grids overlap and the later one only waits).  Both are no-ops for a launch
// without the attribute.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// E2M1 codes of the three balanced base-8 digits of an INT8 code q =
// 64*a + 8*b + c (a in [-2, 2], b and c in [-4, 3]): a | b << 4 | c << 8.  A
// digit d has code 0, 2, 4, 5, 6 for |d| = 0..4 (nibbles packed in 0x65420)
// with the sign in bit 3.  Both digit-plane writers build a 256-entry table
// from it.
__device__ __forceinline__ uint32_t digit_codes(int q) {
    const int c0 = ((q + 4) & 7) - 4;
    const int q1 = (q - c0) >> 3;
    const int b0 = ((q1 + 4) & 7) - 4;
    const int a0 = (q1 - b0) >> 3;
    auto code = [](int d) -> uint32_t {
        const uint32_t mag = (0x65420u >> (4 * (d < 0 ? -d : d))) & 0xFu;
        return d < 0 ? (8u | mag) : mag;
    };
    return code(a0) | code(b0) << 4 | code(c0) << 8;
}

template <class T>
__device__ __forceinline__ T warp_max(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <class T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace moe
