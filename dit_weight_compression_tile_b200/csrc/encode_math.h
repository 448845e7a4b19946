// Arithmetic of the encoder shared by the host compressor (host_encode.cpp) and the device
// compressor (device_encode.cu): quantization resolution and row factors, the E8 nearest point,
// the per-block symbols and their hybrid-integer tokens, FP8 E4M3 rounding.  Every floating-point
// step is one IEEE operation rounded to nearest; device code spells them as __d*_rn intrinsics so
// that no multiply-add is fused, and the host build disables contraction, so both sides produce
// the same bits.
#pragma once
#include <cfloat>
#include <cmath>
#include <cstdint>

#include "format.h"

#if defined(__CUDACC__)
#define EP_HD __host__ __device__
#else
#define EP_HD
#endif

namespace ep {

EP_HD inline double dmul(double a, double b) {
#if defined(__CUDA_ARCH__)
    return __dmul_rn(a, b);
#else
    return a * b;
#endif
}
EP_HD inline double dadd(double a, double b) {
#if defined(__CUDA_ARCH__)
    return __dadd_rn(a, b);
#else
    return a + b;
#endif
}
EP_HD inline double dsub(double a, double b) {
#if defined(__CUDA_ARCH__)
    return __dsub_rn(a, b);
#else
    return a - b;
#endif
}
EP_HD inline double ddiv(double a, double b) {
#if defined(__CUDA_ARCH__)
    return __ddiv_rn(a, b);
#else
    return a / b;
#endif
}
EP_HD inline double dround(double a) {  // nearest integer, ties to even
#if defined(__CUDA_ARCH__)
    return rint(a);
#else
    return std::nearbyint(a);
#endif
}
// exact helpers, spelled per side
#if defined(__CUDA_ARCH__)
__device__ inline double dabs(double a) { return fabs(a); }
__device__ inline double dldexp(double a, int e) { return ldexp(a, e); }
__device__ inline bool f_isinf(float f) { return isinf(f); }
__device__ inline bool f_signbit(float f) { return signbit(f); }
#else
inline double dabs(double a) { return std::fabs(a); }
inline double dldexp(double a, int e) { return std::ldexp(a, e); }
inline bool f_isinf(float f) { return std::isinf(f); }
inline bool f_signbit(float f) { return std::signbit(f); }
#endif

// ------------------------------------------------------------------ resolution and row factors
// q(k) = (64 + k mod 64) 2^(floor(k / 64) - 14), exact in binary floating point
EP_HD inline double q_value(int k) { return dldexp(double(64 + (k % 64)), k / 64 - 14); }

EP_HD inline float factor_of(float rms, int k) {
    if (rms == 0.0f) return 0.0f;
    float f = float(ddiv(double(rms), dmul(2.0, q_value(k))));
    return f_isinf(f) ? FLT_MAX : f;
}

// ------------------------------------------------------------------ E8 nearest point
// nearest point of D8 (Conway & Sloane): round, then repair an odd coordinate sum at the
// coordinate with the largest rounding error (lowest index on ties), moving it towards y
EP_HD inline void nearest_d8(const double *y, double *r) {
    long long s = 0;
    for (int i = 0; i < 8; ++i) {
        r[i] = dround(y[i]);
        s += static_cast<long long>(r[i]);
    }
    if (s & 1) {
        int worst = 0;
        double werr = dabs(dsub(y[0], r[0]));
        for (int i = 1; i < 8; ++i) {
            double e = dabs(dsub(y[i], r[i]));
            if (e > werr) {
                werr = e;
                worst = i;
            }
        }
        r[worst] = dadd(r[worst], (y[worst] < r[worst]) ? -1.0 : 1.0);
    }
}

// v = 2 * nearest point of E8 = D8 u (D8 + 1/2); a distance tie keeps the integer coset
EP_HD inline void quantize_e8(const double *x, int32_t *v) {
    double a[8], b[8], ra[8], rb[8];
    for (int i = 0; i < 8; ++i) {
        a[i] = x[i];
        b[i] = dsub(x[i], 0.5);
    }
    nearest_d8(a, ra);
    nearest_d8(b, rb);
    double da = 0.0, db = 0.0;
    for (int i = 0; i < 8; ++i) da = dadd(da, dmul(dsub(a[i], ra[i]), dsub(a[i], ra[i])));
    for (int i = 0; i < 8; ++i) db = dadd(db, dmul(dsub(b[i], rb[i]), dsub(b[i], rb[i])));
    if (db < da) {
        for (int i = 0; i < 8; ++i) v[i] = int32_t(rb[i]) * 2 + 1;
    } else {
        for (int i = 0; i < 8; ++i) v[i] = int32_t(ra[i]) * 2;
    }
}

// ------------------------------------------------------------------ symbols and tokens
EP_HD inline uint32_t zz(int32_t y) { return y < 0 ? uint32_t(-int64_t(y)) * 2u - 1u : uint32_t(y) * 2u; }

EP_HD inline int bitlen(uint32_t u) {
#if defined(__CUDA_ARCH__)
    return 32 - __clz(u);
#else
    return u ? 32 - __builtin_clz(u) : 0;
#endif
}

// Contexts and coded values of one block, in coding order.  c = v0 mod 2, y_i = (v_i - c) / 2,
// p = parity of y0 + ... + y6.  Coordinate 0: context 0, value 4 zz(a0) + r0 with v0 = 4 a0 + r0;
// coordinates 1..6: context 1 + c, value 2 zz(a) + b with y = 2 a + b; coordinate 7: context
// 3 + 2c + p, value zz((y7 - p) / 2).  Arithmetic shifts are floor divisions here.
EP_HD inline void symbols_of(const int32_t *v, uint8_t *ctx, uint32_t *s) {
    int32_t c = v[0] & 1;
    int32_t par = ((v[0] - c) >> 1) & 1;
    ctx[0] = 0;
    s[0] = 4u * zz(v[0] >> 2) + uint32_t(v[0] & 3);
    for (int i = 1; i < 7; ++i) {
        int32_t y = (v[i] - c) >> 1;
        par ^= y & 1;
        ctx[i] = uint8_t(1 + c);
        s[i] = 2u * zz(y >> 1) + uint32_t(y & 1);
    }
    int32_t y7 = (v[7] - c) >> 1;
    ctx[7] = uint8_t(3 + 2 * c + par);
    s[7] = zz((y7 - par) >> 1);
}

struct Token {
    uint32_t tok, nbits, extra;
};

// hybrid-integer token of s with split m, keeping the `low` low bits of s in the token and two
// bits below the leading one; the bits in between are raw extra bits
EP_HD inline Token token_of(uint32_t s, uint32_t m, uint32_t low) {
    if (s < (1u << m)) return {s, 0, 0};
    uint32_t n = uint32_t(bitlen(s)) - 1;
    uint32_t nbits = n - kTopBits - low;
    uint32_t top = (s >> (n - kTopBits)) & ((1u << kTopBits) - 1u);
    uint32_t tok = (1u << m) + (((((n - m) << kTopBits) | top) << low) | (s & ((1u << low) - 1u)));
    return {tok, nbits, (s >> low) & ((1u << nbits) - 1u)};
}

// ------------------------------------------------------------------ FP8 E4M3 codes
// non-negative finite E4M3 value of code c in [0, 126]
EP_HD inline double e4m3_value(int c) {
    int e = c >> 3, m = c & 7;
    return e == 0 ? dldexp(double(m), -9) : dldexp(1.0 + double(m) / 8.0, e - 7);
}

// round t to the E4M3 grid, nearest with ties to the even code, saturating at 448
EP_HD inline double e4m3_round(float t) {
    double a = dabs(double(t)), r;
    if (a >= e4m3_value(126)) {
        r = e4m3_value(126);
    } else {
        int lo = 0, hi = 126;  // e4m3_value(lo) <= a < e4m3_value(hi)
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (e4m3_value(mid) <= a)
                lo = mid;
            else
                hi = mid;
        }
        double dlo = dsub(a, e4m3_value(lo)), dhi = dsub(e4m3_value(hi), a);
        if (dlo < dhi)
            r = e4m3_value(lo);
        else if (dhi < dlo)
            r = e4m3_value(hi);
        else
            r = (lo % 2 == 0) ? e4m3_value(lo) : e4m3_value(hi);
    }
    return f_signbit(t) ? -r : r;
}

}  // namespace ep
