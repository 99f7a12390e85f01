// CPU oracle of the routed FP4 mixture-of-experts layer.
//
// TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
// load this file: it is used by tests/, by the smoke check and by the
// CPU-baseline leg of the benchmark.  It shares no code, header, table or
// constant with the CUDA library; the two meet only at the seeded input
// generator (synth/), which holds none of the layer's arithmetic.
//
// Source of the method.  "DeepSeek-V4-Flash on AMD gfx90a: Correctness
// Recovery and Inference Performance Engineering" (abstract) names the steps:
// FP4 routed mixture-of-experts with packed FP4 expert weights, INT8
// activation quantisation, expert sorting before the expert GEMMs, and the W2
// projection whose layout bug permuted outputs.  The blog post "DeepSeek V4
// Flash on 8x R9600D" (model facts paragraph) fixes 256 routed experts with 6
// active per token.  The pages give no formulas; every formula below is the
// plain reading of those names; each such reading is stated where it is used.
//
// Plainness rules: every value is computed from its definition, one output at
// a time, in fp64 where the definition is real-valued; fp32 only where the
// definition itself rounds to fp32 (quantisation scales, G/h/Y).  No blocking,
// fusion or reordering beyond grouping independent pairs across threads.
//
// Exactness domain of the expert dot products: every term q * w is exact in
// fp64 and, for scale bytes of one row spanning at most ~28 binades, so is
// every partial sum (the int64 fixed-point variant below checks this).
//
// Pins (tests/): E2M1 and E8M0 decode against ml_dtypes; route against a full
// stable sort; sort against numpy's stable argsort; quantisation special
// cases; exp against libm within 2 ulp; dot products fp64 vs int64 and vs a
// float64 matmul in the integer special case; the layer against a dense-mask
// brute force, token-order invariance and the E=1, k=1 plain MLP.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---- Reading: FP4 is OCP MX E2M1 ("FP4").  1 sign, 2 exponent bits (bias 1), 1 mantissa
// bit; exponent 0 is subnormal (0.5 * m).  No NaN/Inf codes; code 8 is -0.
double e2m1_value(int code) {
    const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

// ---- Reading: one UE8M0 scale per 32 input-dimension elements: 2^(s-127);
// 255 is NaN and rejected by the callers.
double e8m0_value(int s) { return std::ldexp(1.0, s - 127); }

// ---- Reading: canonical nibble order: byte j of a row holds element 2j in its low
// nibble and element 2j+1 in its high nibble.
inline int code_at(const uint8_t* row_codes, int k) {
    const uint8_t b = row_codes[k >> 1];
    return (k & 1) ? (b >> 4) : (b & 15);
}

// Weight element w[n,k] = e2m1(code) * 2^(S[n, k/32] - 127).
inline double weight_at(const uint8_t* row_codes, const uint8_t* row_scales, int k) {
    return e2m1_value(code_at(row_codes, k)) * e8m0_value(row_scales[k / 32]);
}

// ---- The layer's fp32 exp (the same specification is implemented separately
// on the GPU so that SwiGLU, and hence the INT8 codes of h, agree bit for bit).  Cody-Waite reduction x = n*ln2 + r with ln2
// split into a 12-significant-bit high part and a low part, degree-7 Taylor
// polynomial of e^r by Horner with fused multiply-adds, then scaling by 2^n
// through the exponent field.  Constants derive from ln 2 and 1/j!, rounded to
// fp32.  All operations are single fp32 roundings (compiled without
// contraction).
const float kLog2e = 1.44269502162933349609375f;   // fp32(1/ln 2)
const float kLn2Hi = 0.693115234375f;              // ln 2 truncated to 12 significant bits
const float kLn2Lo = 3.19461832987144589424133e-05f; // fp32(ln 2 - kLn2Hi)
const float kInvFact[8] = {1.0f, 1.0f, 0.5f, 0.16666667163372039794921875f,
                           0.041666667908430099487304688f, 0.0083333337679505348205566406f,
                           0.0013888889225199818611145020f, 0.00019841270113829523324966431f};

float pow2_float(int n) {  // 2^n for n in [-126, 127], built from the exponent field
    uint32_t bits = (uint32_t)(n + 127) << 23;
    float f;
    std::memcpy(&f, &bits, 4);
    return f;
}

float layer_exp(float x) {
    if (x != x) return x;
    if (x > 88.8f) return INFINITY;
    if (x < -104.0f) return 0.0f;
    const float nf = std::nearbyint(x * kLog2e);
    float r = std::fma(-nf, kLn2Hi, x);
    r = std::fma(-nf, kLn2Lo, r);
    float p = kInvFact[7];
    for (int j = 6; j >= 0; --j) p = std::fma(p, r, kInvFact[j]);
    const int n = (int)nf;
    if (n > 126) return (p * pow2_float(n - 1)) * 2.0f;
    if (n < -125) return (p * pow2_float(n + 100)) * pow2_float(-100);
    return p * pow2_float(n);
}

// ---- SwiGLU between W1 and W2 (no clamp or limit on g or u):
// h = fp32( fp32(g / fp32(1 + exp(-g))) * u ).
float swiglu(float g, float u) {
    const float d = 1.0f + layer_exp(-g);
    const float sg = g / d;
    return sg * u;
}

// ---- Reading: INT8 activation quantisation is per row (token for x, pair for
// h) and symmetric.  a = max|v| (exact), scale
// s = fp32(a / 127) by IEEE division, q = clamp(round-half-even(fp32(v / s)),
// -127, 127); an all-zero row gives s = 0, q = 0.
void quant_row(const float* v, int n, int8_t* q, float* s_out) {
    float a = 0.0f;
    for (int i = 0; i < n; ++i) a = std::max(a, std::fabs(v[i]));
    const float s = a / 127.0f;
    *s_out = s;
    for (int i = 0; i < n; ++i) {
        if (a == 0.0f) { q[i] = 0; continue; }
        float r = std::nearbyint(v[i] / s);
        r = std::min(127.0f, std::max(-127.0f, r));
        q[i] = (int8_t)r;
    }
}

// ---- expert dot product: sum_k q[k] * w[n,k] over one weight row, fp64,
// ascending k.  Every term is exact in fp64 (int8 * 3-bit significand * 2^e).
double row_dot(const int8_t* q, const uint8_t* row_codes, const uint8_t* row_scales, int K) {
    double acc = 0.0;
    for (int k = 0; k < K; ++k) acc += (double)q[k] * weight_at(row_codes, row_scales, k);
    return acc;
}

// Second, independent reference of the same sum: int64 fixed point in units of
// 2^(Smin - 128), Smin = smallest scale byte of the row; 2*e2m1 is an integer
// in [-12, 12].  Returns false when the shift range would overflow int64.
int twice_e2m1_int(int code) {
    static const int mag[8] = {0, 1, 2, 3, 4, 6, 8, 12};
    return (code & 8) ? -mag[code & 7] : mag[code & 7];
}

bool row_dot_fixed(const int8_t* q, const uint8_t* row_codes, const uint8_t* row_scales, int K,
                   double* out) {
    int smin = 255;
    for (int b = 0; b < K / 32; ++b) smin = std::min(smin, (int)row_scales[b]);
    int64_t acc = 0;
    for (int k = 0; k < K; ++k) {
        const int sh = row_scales[k / 32] - smin;
        if (sh > 40) return false;
        acc += (int64_t)q[k] * twice_e2m1_int(code_at(row_codes, k)) * (int64_t(1) << sh);
    }
    if (acc >= (int64_t(1) << 53) || acc <= -(int64_t(1) << 53)) return false;
    *out = std::ldexp((double)acc, smin - 128);
    return true;
}

// ---- Routing.  Top-k experts by logit, descending, ties to the lower
// expert id, NaN below every number.  Softmax is monotone, so the top-k of the
// probabilities is the top-k of the logits.  Gates renormalise the softmax over
// the k chosen experts; the full-softmax denominator cancels; there is
// no routed scaling factor.
bool beats(float a, int ia, float b, int ib) {
    const bool na = a != a, nb = b != b;
    if (na || nb) return (na && nb) ? ia < ib : nb;
    if (a != b) return a > b;
    return ia < ib;
}

void route_token(const float* l, int E, int k, int32_t* idx, double* gates) {
    std::vector<char> taken(E, 0);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || beats(l[e], e, l[best], best)) best = e;
        }
        taken[best] = 1;
        idx[j] = best;
    }
    const double lmax = (double)l[idx[0]];
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += std::exp((double)l[idx[j]] - lmax);
    for (int j = 0; j < k; ++j) gates[j] = std::exp((double)l[idx[j]] - lmax) / den;
}

// bf16 round-to-nearest-even of a double (round-to-odd into fp32 first, which
// makes the second rounding exact), returned as raw bits.
uint16_t bf16_from_double(double v) {
    if (v != v) return 0x7FC0;
    float f = (float)v;
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if (std::isfinite(f) && (double)f != v) {
        if (std::fabs((double)f) > std::fabs(v)) u -= 1;  // toward zero
        u |= 1;                                           // sticky (round to odd)
    }
    if ((u & 0x7F800000u) == 0x7F800000u) return (uint16_t)(u >> 16);  // inf
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

float bf16_bits_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

template <class F>
void parallel_for(int64_t n, int nthreads, F f) {
    nthreads = std::max(1, std::min<int>(nthreads, 256));
    if (n <= 1 || nthreads == 1) {
        for (int64_t i = 0; i < n; ++i) f(i);
        return;
    }
    std::vector<std::thread> th;
    std::atomic<int64_t> next{0};
    for (int t = 0; t < nthreads; ++t)
        th.emplace_back([&] {
            for (int64_t i; (i = next.fetch_add(1)) < n;) f(i);
        });
    for (auto& x : th) x.join();
}

struct Dims {
    int T, H, I, E, k;
};

// One pair's expert MLP, steps 5-8 of the definition, for token activation
// (xq, sx) through expert e.  Writes hq[I], sh, Y[H] (fp32).
void expert_pair(const Dims& d, const int8_t* xq, float sx, int e, const uint8_t* w1c,
                 const uint8_t* w1s, const uint8_t* w2c, const uint8_t* w2s, int8_t* hq, float* sh,
                 float* Y) {
    const int H = d.H, I = d.I;
    std::vector<float> h(I);
    const uint8_t* c1 = w1c + (int64_t)e * 2 * I * (H / 2);
    const uint8_t* s1 = w1s + (int64_t)e * 2 * I * (H / 32);
    for (int i = 0; i < I; ++i) {
        // Step 5 (W1; reading: rows [0,I) are gate, [I,2I) up): G = fp32(fp64(sx) * exact sum).
        const double dg = row_dot(xq, c1 + (int64_t)i * (H / 2), s1 + (int64_t)i * (H / 32), H);
        const double du =
            row_dot(xq, c1 + (int64_t)(I + i) * (H / 2), s1 + (int64_t)(I + i) * (H / 32), H);
        const float g = (float)((double)sx * dg);
        const float u = (float)((double)sx * du);
        h[i] = swiglu(g, u);  // step 6
    }
    quant_row(h.data(), I, hq, sh);  // step 7
    const uint8_t* c2 = w2c + (int64_t)e * H * (I / 2);
    const uint8_t* s2 = w2s + (int64_t)e * H * (I / 32);
    for (int n = 0; n < H; ++n) {  // step 8 (W2)
        const double dy = row_dot(hq, c2 + (int64_t)n * (I / 2), s2 + (int64_t)n * (I / 32), I);
        Y[n] = (float)((double)*sh * dy);
    }
}

}  // namespace

extern "C" {

double orc_e2m1(int code) { return e2m1_value(code & 15); }
double orc_e8m0(int s) { return e8m0_value(s); }
float orc_exp(float x) { return layer_exp(x); }
float orc_swiglu(float g, float u) { return swiglu(g, u); }
uint16_t orc_bf16_from_double(double v) { return bf16_from_double(v); }

void orc_exp_array(const float* x, float* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = layer_exp(x[i]);
}

void orc_quant_rows(const float* v, int64_t rows, int cols, int8_t* q, float* s) {
    for (int64_t r = 0; r < rows; ++r) quant_row(v + r * cols, cols, q + r * cols, s + r);
}

// x: raw bf16 bits [T, H] -> xq [T, H], sx [T] (step 4 of the definition).
void orc_quant_x(const uint16_t* x, int T, int H, int8_t* xq, float* sx, int nthreads) {
    parallel_for(T, nthreads, [&](int64_t t) {
        std::vector<float> v(H);
        for (int h = 0; h < H; ++h) v[h] = bf16_bits_to_float(x[t * H + h]);
        quant_row(v.data(), H, xq + t * H, sx + t);
    });
}

// Step 1, the router projection in front of the path (the layer takes its
// logits as an input; this is the reference for the router kernel).  Reading:
// the router is a plain linear map of the bf16 activations with fp32 weights,
// one logit per routed expert ("DeepSeek V4 Flash on 8x R9600D", model facts:
// 256 routed experts):
//   S[t, e] = sum_h x[t, h] * Wr[e, h] + b[e],
// in fp64, h in ascending order, x decoded from bf16 exactly, b optional (NULL
// = no bias).  x: raw bf16 bits [T, H]; Wr [E, H] fp32; out [T, E] fp64.
void orc_router_logits(const uint16_t* x, const float* wr, const float* bias, int T, int H, int E, double* out,
                       int nthreads) {
    parallel_for((int64_t)T * E, nthreads, [&](int64_t te) {
        const int64_t t = te / E, e = te % E;
        double s = 0.0;
        for (int h = 0; h < H; ++h) s += (double)bf16_bits_to_float(x[t * H + h]) * (double)wr[e * H + h];
        out[te] = bias ? s + (double)bias[e] : s;
    });
}

void orc_route(const float* logits, int T, int E, int k, int32_t* idx, double* gates) {
    for (int t = 0; t < T; ++t)
        route_token(logits + (int64_t)t * E, E, k, idx + (int64_t)t * k, gates + (int64_t)t * k);
}

// Step 3: stable counting sort (reading: ascending pair id inside an expert) of pair ids p = t*k + j by expert.
// Returns 0, or -1 when an expert id is outside [0, E).
int orc_sort(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets,
             int32_t* perm, int32_t* pos) {
    const int64_t P = (int64_t)T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < P; ++p) {
        if (idx[p] < 0 || idx[p] >= E) return -1;
        counts[idx[p]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    std::vector<int32_t> fill(offsets, offsets + E);
    for (int64_t p = 0; p < P; ++p) {
        const int32_t i = fill[idx[p]]++;
        perm[i] = (int32_t)p;
        pos[p] = i;
    }
    return 0;
}

double orc_row_dot(const int8_t* q, const uint8_t* codes, const uint8_t* scales, int K) {
    return row_dot(q, codes, scales, K);
}

int orc_row_dot_fixed(const int8_t* q, const uint8_t* codes, const uint8_t* scales, int K,
                      double* out) {
    return row_dot_fixed(q, codes, scales, K, out) ? 0 : 1;
}

// Many rows at once: out[r] = row_dot(q[r % nq... ]) -- q row qi[r], weight row wi[r].
void orc_rows_dot(const int8_t* q, int K, const int32_t* qrow, const uint8_t* codes,
                  const uint8_t* scales, const int64_t* wrow, int64_t n, double* out,
                  double* out_fixed, int32_t* fixed_ok, int nthreads) {
    parallel_for(n, nthreads, [&](int64_t r) {
        const int8_t* qq = q + (int64_t)qrow[r] * K;
        const uint8_t* c = codes + wrow[r] * (K / 2);
        const uint8_t* s = scales + wrow[r] * (K / 32);
        out[r] = row_dot(qq, c, s, K);
        if (out_fixed) fixed_ok[r] = row_dot_fixed(qq, c, s, K, &out_fixed[r]) ? 1 : 0;
    });
}

// The whole layer (steps 2-9) for every token.  Outputs are in natural
// order: idx/gates [T,k]; counts [E]; offsets [E+1]; perm/pos [P]; xq [T,H];
// sx [T]; hq [P,I] and sh [P] indexed by pair id p = t*k + j; Y [P,H] fp32
// (may be NULL); y [T,H] raw bf16 bits.  Returns 0, or -1 on a bad argument.
int orc_forward(int T, int H, int I, int E, int k, const uint16_t* x, const float* logits,
                const uint8_t* w1c, const uint8_t* w1s, const uint8_t* w2c, const uint8_t* w2s,
                int32_t* idx, double* gates, int32_t* counts, int32_t* offsets, int32_t* perm,
                int32_t* pos, int8_t* xq, float* sx, int8_t* hq, float* sh, float* Y,
                uint16_t* y, int nthreads) {
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || H % 32 || I % 32) return -1;
    const Dims d{T, H, I, E, k};
    const int64_t P = (int64_t)T * k;
    orc_route(logits, T, E, k, idx, gates);                        // step 2
    if (orc_sort(idx, T, k, E, counts, offsets, perm, pos)) return -1;  // step 3
    orc_quant_x(x, T, H, xq, sx, nthreads);                        // step 4
    std::vector<float> Yown;
    if (!Y) {
        Yown.resize((size_t)P * H);
        Y = Yown.data();
    }
    // steps 5-8, one pair at a time, in sorted (expert-grouped) order
    parallel_for(P, nthreads, [&](int64_t i) {
        const int64_t p = perm[i];
        const int64_t t = p / k;
        expert_pair(d, xq + t * H, sx[t], idx[p], w1c, w1s, w2c, w2s, hq + p * I, sh + p, Y + p * H);
    });
    // step 9: y[t,n] = bf16( sum_j gates[t,j] * Y[pair (t,j)][n] ), fp64, slot order
    parallel_for(T, nthreads, [&](int64_t t) {
        for (int n = 0; n < H; ++n) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) acc += gates[t * k + j] * (double)Y[(t * k + j) * H + n];
            y[t * H + n] = bf16_from_double(acc);
        }
    });
    return 0;
}

// The layer for a subset of tokens only (every value of those tokens is the
// same as in orc_forward).  tok[ntok]; outputs indexed by position in `tok`:
// idx/gates [ntok,k], xq [ntok,H], sx [ntok], hq [ntok*k, I], sh [ntok*k],
// y [ntok, H].  Used for sampled checks at full size.
int orc_forward_tokens(int T, int H, int I, int E, int k, const uint16_t* x, const float* logits,
                       const uint8_t* w1c, const uint8_t* w1s, const uint8_t* w2c,
                       const uint8_t* w2s, const int32_t* tok, int ntok, int32_t* idx,
                       double* gates, int8_t* xq, float* sx, int8_t* hq, float* sh, uint16_t* y,
                       int nthreads) {
    if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || H % 32 || I % 32) return -1;
    for (int i = 0; i < ntok; ++i)
        if (tok[i] < 0 || tok[i] >= T) return -1;
    const Dims d{T, H, I, E, k};
    for (int i = 0; i < ntok; ++i)
        route_token(logits + (int64_t)tok[i] * E, E, k, idx + (int64_t)i * k, gates + (int64_t)i * k);
    parallel_for(ntok, nthreads, [&](int64_t i) {
        std::vector<float> v(H);
        for (int h = 0; h < H; ++h) v[h] = bf16_bits_to_float(x[(int64_t)tok[i] * H + h]);
        quant_row(v.data(), H, xq + i * H, sx + i);
    });
    std::vector<float> Y((size_t)ntok * k * H);
    parallel_for((int64_t)ntok * k, nthreads, [&](int64_t q) {
        const int64_t i = q / k;
        expert_pair(d, xq + i * H, sx[i], idx[q], w1c, w1s, w2c, w2s, hq + q * I, sh + q,
                    Y.data() + q * H);
    });
    for (int64_t i = 0; i < ntok; ++i)
        for (int n = 0; n < H; ++n) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) acc += gates[i * k + j] * (double)Y[(i * k + j) * H + n];
            y[i * H + n] = bf16_from_double(acc);
        }
    return 0;
}

// Brute force: every token through EVERY expert, combined with a dense
// gate mask (gate of the slot that chose the expert, else 0), summed in fp64
// in expert order.  No sort, no gather.  y_f64 [T,H] before rounding, y [T,H].
int orc_forward_dense(int T, int H, int I, int E, int k, const uint16_t* x, const float* logits,
                      const uint8_t* w1c, const uint8_t* w1s, const uint8_t* w2c,
                      const uint8_t* w2s, double* y_f64, uint16_t* y, int nthreads) {
    if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || k > E || H % 32 || I % 32) return -1;
    const Dims d{T, H, I, E, k};
    parallel_for(T, nthreads, [&](int64_t t) {
        std::vector<int32_t> idx(k);
        std::vector<double> gates(k);
        route_token(logits + t * E, E, k, idx.data(), gates.data());
        std::vector<double> mask(E, 0.0);
        for (int j = 0; j < k; ++j) mask[idx[j]] = gates[j];
        std::vector<float> v(H);
        std::vector<int8_t> xq(H);
        float sx;
        for (int h = 0; h < H; ++h) v[h] = bf16_bits_to_float(x[t * H + h]);
        quant_row(v.data(), H, xq.data(), &sx);
        std::vector<double> acc(H, 0.0);
        std::vector<int8_t> hq(I);
        std::vector<float> Y(H);
        for (int e = 0; e < E; ++e) {
            float sh;
            expert_pair(d, xq.data(), sx, e, w1c, w1s, w2c, w2s, hq.data(), &sh, Y.data());
            for (int n = 0; n < H; ++n) acc[n] += mask[e] * (double)Y[n];
        }
        for (int n = 0; n < H; ++n) {
            y_f64[t * H + n] = acc[n];
            y[t * H + n] = bf16_from_double(acc[n]);
        }
    });
    return 0;
}

}  // extern "C"
