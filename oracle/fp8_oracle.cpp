// CPU oracle of the FP8 block-quantised dense projection.
//
// TEST INFRASTRUCTURE ONLY, like moe_oracle.cpp: used by tests/, never by the
// product path; it shares no code with the CUDA library.
//
// Source of the method.  "DeepSeek-V4-Flash on AMD gfx90a: Correctness
// Recovery and Inference Performance Engineering" (abstract) runs the model's
// dense projections in FP8; "DeepSeek V4 Flash on 8x R9600D" (model facts
// paragraph) names the format "FP8 block quantization".  The pages give no
// formula.  Readings (plainest consistent with those words and with the MXFP4
// experts of the same model, whose block scales are UE8M0 powers of two):
//   F1  FP8 is OCP E4M3 (E4M3FN): 1 sign, 4 exponent bits (bias 7), 3 mantissa
//       bits; exponent 0 is subnormal (m/8 * 2^-6); 0x7F / 0xFF are NaN; the
//       largest finite magnitude is 448.
//   F2  Weight blocks are 128 x 128 (output rows x inputs) with one scale per
//       block; activation blocks are 1 x 128 (one token, 128 consecutive
//       inputs).  Every scale is a power of two stored as a UE8M0 byte:
//       value 2^(byte - 127).
//   F3  Activation quantisation of a block with a = max |x| (exact, bf16
//       inputs): the scale is the smallest power of two 2^e with a <= 448 * 2^e
//       (so no code saturates), byte e + 127 clamped to [0, 254]; codes are
//       x / 2^e rounded to the nearest E4M3 value, ties to even.  An all-zero
//       block has byte 0 and all codes 0.
//   F4  y[t, n] = bf16_rne( sum_k xq[t,k] 2^(sx[t,k/128]-127) *
//       wq[n,k] 2^(sw[n/128,k/128]-127) ), the sum taken in fp64.
// Every product of two E4M3 values times two powers of two is exact in fp64.
#include <cmath>
#include <cstdint>
#include <thread>
#include <vector>

// nearest bf16 of a double (pinned with the rest of moe_oracle.cpp)
extern "C" uint16_t orc_bf16_from_double(double v);

namespace {

double e4m3_value(int code) {
    const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return std::nan("");
    const double mag = e == 0 ? std::ldexp((double)m, -9) : std::ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

// Nearest E4M3 code of v (|v| <= 448), ties to the even code (even mantissa):
// the candidates are the finite codes bracketing |v|, found by scanning the
// 127 non-negative finite magnitudes in order.
int e4m3_code_rne(double v) {
    const int sign = std::signbit(v) ? 0x80 : 0;
    const double a = std::fabs(v);
    int best = 0;
    for (int c = 1; c <= 0x7E; ++c) {   // magnitudes increase with the code
        if (e4m3_value(c) <= a) best = c;
        else break;
    }
    if (best < 0x7E) {
        const double lo = e4m3_value(best), hi = e4m3_value(best + 1);
        const double dl = a - lo, dh = hi - a;
        if (dh < dl || (dh == dl && ((best + 1) & 1) == 0)) best = best + 1;
    }
    return sign | best;
}

double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    static_assert(sizeof(f) == 4, "fp32");
    __builtin_memcpy(&f, &u, 4);
    return (double)f;
}

template <class F>
void parallel_for(int64_t n, int nthreads, F f) {
    if (nthreads <= 1 || n < 64) {
        for (int64_t i = 0; i < n; ++i) f(i);
        return;
    }
    std::vector<std::thread> th;
    for (int w = 0; w < nthreads; ++w)
        th.emplace_back([=]() {
            for (int64_t i = w; i < n; i += nthreads) f(i);
        });
    for (auto& t : th) t.join();
}

}  // namespace

extern "C" {

double orc_e4m3(int code) { return e4m3_value(code); }
int orc_e4m3_code(double v) { return e4m3_code_rne(v); }

// F3: x raw bf16 bits [T, K] -> q [T, K] E4M3 codes, s [T, K/128] UE8M0 bytes.
void orc_fp8_quant_act(const uint16_t* x, int T, int K, uint8_t* q, uint8_t* s, int nthreads) {
    const int G = K / 128;
    parallel_for((int64_t)T * G, nthreads, [&](int64_t tg) {
        const int64_t t = tg / G, g = tg % G;
        const uint16_t* xr = x + t * K + g * 128;
        double a = 0.0;
        for (int j = 0; j < 128; ++j) a = std::fmax(a, std::fabs(bf16_to_double(xr[j])));
        if (a == 0.0) {
            s[tg] = 0;
            for (int j = 0; j < 128; ++j) q[t * K + g * 128 + j] = 0;
            return;
        }
        int e = -127;  // smallest e with a <= 448 * 2^e (exact comparisons)
        while (a > 448.0 * std::ldexp(1.0, e)) ++e;
        if (e > 127) e = 127;
        s[tg] = (uint8_t)(e + 127);
        for (int j = 0; j < 128; ++j)
            q[t * K + g * 128 + j] = (uint8_t)e4m3_code_rne(std::ldexp(bf16_to_double(xr[j]), -e));
    });
}

// F4: y[t, n] for tokens [0, T) from q/s (F3) and the weights wq [N, K],
// ws [N/128, K/128].  y_bf16 [T, N] (raw bits), y64 [T, N] (the fp64 sum) and
// yabs [T, N] (the sum of |terms|, for error bounds); y64 / yabs may be NULL.
void orc_fp8_linear(const uint8_t* q, const uint8_t* s, const uint8_t* wq, const uint8_t* ws, int T, int N, int K,
                    uint16_t* y_bf16, double* y64, double* yabs, int nthreads) {
    const int G = K / 128;
    parallel_for((int64_t)T * N, nthreads, [&](int64_t tn) {
        const int64_t t = tn / N, n = tn % N;
        double acc = 0.0, aabs = 0.0;
        for (int k = 0; k < K; ++k) {
            const double xv = std::ldexp(e4m3_value(q[t * K + k]), (int)s[t * G + k / 128] - 127);
            const double wv = std::ldexp(e4m3_value(wq[n * K + k]), (int)ws[(n / 128) * G + k / 128] - 127);
            acc += xv * wv;
            aabs += std::fabs(xv * wv);
        }
        y_bf16[tn] = orc_bf16_from_double(acc);
        if (y64) y64[tn] = acc;
        if (yabs) yabs[tn] = aabs;
    });
}

}  // extern "C"
