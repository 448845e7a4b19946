/*
 * Oracle for the lattice-rANS tile stream -- TEST INFRASTRUCTURE ONLY.
 * See ep_oracle.h for scope.  Build: gcc -std=c99 -O2 -ffp-contract=off -fPIC -shared.
 *
 * Sources followed (page title, section):
 *   [ABS]  "EntroPack: Fast and Accurate Entropy-Coded Weight Compression at Arbitrary
 *          Bitrates", Abstract -- row-normalized E8 lattice quantization, conditional
 *          model of lattice coordinates, sampled storage estimates pick the resolution,
 *          entropy coding in tiles that decode on their own, fused decode + reconstruction,
 *          BF16 / FP16 / FP8 / INT8 containers.
 *   [API]  "EntroPack API reference", compress / CompressedTensor -- non-empty 2-D finite
 *          input, actual_bpp = 8 * storage_nbytes / numel including metadata.
 *   [README] "EntroPack README", Get started / Configuration -- target range [0.001, 11].
 *   [LIN]  "Compressed Linear usage", Combine compression with FP8 or INT8 computation --
 *          lossy compression applied to FP8/INT8 weight codes, target < 8, per-row scales
 *          counted in storage.
 * Textbook material restated here (not from the pages):
 *   Conway & Sloane, "Fast quantizing and decoding algorithms for lattice quantizers and
 *   codes" (IEEE Trans. IT, 1982): nearest point of D_n and of E8 = D8 u (D8 + 1/2).
 *   Duda, "Asymmetric numeral systems" (2013): range variant rANS.
 *   Giesen, "Interleaved entropy coders" (2014): several rANS states sharing one stream.
 *   Micikevicius et al., "FP8 Formats for Deep Learning" (2022): E4M3 encoding.
 */
#include "ep_oracle.h"

#include <float.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------
 * Stream constants (format version 4).  These are the build's readings of what the
 * pages leave open: 11-bit frequency tables (every frequency below 2^11), 32-bit states
 * with 16-bit renormalisation words, 32 interleaved states per tile, seven coding
 * contexts, hybrid-integer tokens with 2 bits below the leading one and a per-context
 * number of low bits kept in the token, raw extra bits in a separate stream per tile,
 * and, when the tokens allow it, coordinates 1..6 coded in pairs (12-bit pair tables).
 * ---------------------------------------------------------------------------------- */
#define MAGIC 0x31545045u /* bytes 'E','P','T','1' */
#define VERSION 4
#define PROB_BITS 11
#define PROB_M 2048u
#define STATE_L 65536u
#define LANES 32
#define NCTX 7
#define H_BITS 2             /* bits below the leading one carried by an escape token */
#define VALUE_BITS 22        /* every symbol value is below 2^22 */
#define HEADER_BYTES 64
#define TILE_HEAD 192        /* 32 states (u32) + 32 word counts (u16) */
#define TILE_BUDGET 5952.0   /* expected payload bytes a tile may hold (a 6 KB staging buffer) */
#define NQ 1280
#define SAMPLE_TARGET 65536

/* low bits of the value kept inside every token, and the largest split, per context:
 * coordinate 0 keeps v0 mod 4 (coset and the parity of y0), coordinates 1..6 keep the parity
 * of y_i, coordinate 7 keeps nothing.  The largest splits keep every directly coded coordinate
 * 0 within -256 <= v0 <= 255 and every directly coded y_i = (v_i - c) / 2 of coordinates 1..7
 * within -256 <= y_i <= 255. */
static const int32_t CTX_LOW[NCTX] = {2, 1, 1, 0, 0, 0, 0};
static const int32_t CTX_MAX_SPLIT[NCTX] = {9, 9, 9, 8, 8, 8, 8};
/* splits up to which every directly coded coordinate v itself lies in [-256, 255] */
static const int32_t CTX_NARROW_SPLIT[NCTX] = {9, 8, 8, 7, 7, 7, 7};

/* Paired coding (a reading of the pages' conditional model, which they leave open): when the
 * tokens of contexts 1 and 2 concentrate below 40, coordinates (1,2), (3,4) and (5,6) of a block
 * are coded as one symbol each.  With A the
 * context's token alphabet length and B = min(A, 40), a pair of tokens both below B is symbol
 * t_a B + t_b of a table of B^2 + 1 symbols summing to 2^12; the last symbol is an escape, taken
 * by pairs with a token at or above B and by pairs seen fewer than N / 2^16 times (N: the
 * context's pair count).  An escaped pair's two tokens follow in the raw bits. */
#define PAIR_BITS 12
#define PAIR_M 4096u
#define PAIR_BASE_MAX 40u           /* largest pair base B */
#define PAIR_MAX_ALPHABET 256u      /* contexts 1 and 2 are paired up to this alphabet length */
#define PAIR_OUTSIDE_SCALE 4096u    /* ... and while at most 1 / 2^12 of their tokens lie beyond the base */
#define PAIR_MIN_BLOCKS (1 << 17)   /* automatic coding pairs tensors of at least this many blocks */
#define PAIR_RARE_SCALE 65536u      /* a pair seen c times is escaped when c * 2^16 < N */

static size_t al16(size_t n) { return (n + 15) & ~(size_t)15; }

/* ---------------------------------- scalar decode of inputs -------------------------- */
static double half_to_double(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return s ? -v : v;
}

static double src_value(const void *src, int32_t dt, int64_t i)
{
    if (dt == ORD_BF16) {
        uint32_t b = (uint32_t)((const uint16_t *)src)[i] << 16;
        float f;
        memcpy(&f, &b, 4);
        return (double)f;
    }
    if (dt == ORD_FP16)
        return half_to_double(((const uint16_t *)src)[i]);
    return (double)((const float *)src)[i];
}

/* ---------------------------------- container conversions --------------------------- */
/* fp32 -> bf16, round to nearest even (finite inputs; overflow rounds to infinity) */
uint16_t or_bf16_from_float(float w)
{
    uint32_t b;
    memcpy(&b, &w, 4);
    if ((b & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((b >> 16) | 0x40);
    b += 0x7fffu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

/* fp32 -> IEEE binary16, round to nearest even, subnormals kept, overflow to infinity.
 * Written from the binary16 definition: value = (-1)^s * 2^(e-15) * 1.m, e in [1,30]. */
uint16_t or_fp16_from_float(float w)
{
    double a = fabs((double)w);
    uint16_t s = signbit(w) ? 0x8000 : 0;
    if (isnan(w))
        return 0x7e00;
    if (a < ldexp(1.0, -14)) { /* subnormal range: multiples of 2^-24 */
        double q = nearbyint(a * ldexp(1.0, 24)); /* exact scaling, then RNE */
        return (uint16_t)(s | (uint16_t)q);        /* q == 1024 is the smallest normal */
    }
    int e;
    double fr = frexp(a, &e); /* a = fr * 2^e, fr in [0.5, 1) */
    double mant = nearbyint(fr * 2048.0);  /* 11 significant bits, RNE */
    if (mant == 2048.0) {
        mant = 1024.0;
        e += 1;
    }
    int be = e - 1 + 15;
    if (be >= 31)
        return (uint16_t)(s | 0x7c00);
    return (uint16_t)(s | (uint16_t)(be << 10) | (uint16_t)((int)mant - 1024));
}

/* fp32 -> FP8 E4M3 (the "FN" variant: no infinities, S.1111.111 is NaN, max 448),
 * round to nearest even, saturating to +-448.  Exponent bias 7, smallest normal 2^-6,
 * subnormal step 2^-9. */
uint8_t or_e4m3_from_float(float w)
{
    double a = fabs((double)w);
    uint8_t s = signbit(w) ? 0x80 : 0;
    if (isnan(w))
        return 0x7f;
    if (a < ldexp(1.0, -6)) {
        double q = nearbyint(a * 512.0); /* multiples of 2^-9 */
        return (uint8_t)(s | (uint8_t)q); /* q == 8 encodes 2^-6 exactly */
    }
    int e;
    double fr = frexp(a, &e);
    double mant = nearbyint(fr * 16.0); /* 4 significant bits */
    if (mant == 16.0) {
        mant = 8.0;
        e += 1;
    }
    int be = e - 1 + 7;
    int mm = (int)mant - 8;
    if (be > 15 || (be == 15 && mm == 7))
        return (uint8_t)(s | 0x7e); /* saturate to 448 */
    return (uint8_t)(s | (uint8_t)(be << 3) | (uint8_t)mm);
}

/* fp32 -> int8 code: round to nearest even, clamp to the symmetric range [-127, 127] */
int8_t or_int8_from_float(float w)
{
    if (w >= 127.0f)
        return 127;
    if (w <= -127.0f)
        return -127;
    return (int8_t)(int)nearbyintf(w);
}

static double e4m3_value(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v = e ? ldexp(8.0 + m, e - 10) : ldexp((double)m, -9);
    return s ? -v : v;
}

void or_convert_batch(const float *w, int64_t n, int32_t dt, void *out)
{
    for (int64_t i = 0; i < n; i++) {
        if (dt == ORD_BF16)
            ((uint16_t *)out)[i] = or_bf16_from_float(w[i]);
        else if (dt == ORD_FP16)
            ((uint16_t *)out)[i] = or_fp16_from_float(w[i]);
        else if (dt == ORD_FP32)
            ((float *)out)[i] = w[i];
        else if (dt == ORD_INT8)
            ((int8_t *)out)[i] = or_int8_from_float(w[i]);
        else
            ((uint8_t *)out)[i] = or_e4m3_from_float(w[i]);
    }
}

static int elt_size(int32_t dt)
{
    return dt == ORD_FP32 ? 4 : (dt == ORD_BF16 || dt == ORD_FP16) ? 2 : 1;
}

/* ---------------------------------- resolution grid ---------------------------------- */
/* Reading: the "quantization resolution" is a lattice scale q on a fixed grid that is
 * exact in binary floating point: q(k) = (64 + k mod 64) / 64 * 2^(floor(k/64) - 8),
 * k in [0, 1280), i.e. q from 2^-8 to just under 2^12 with 64 linear steps per octave. */
double or_q_of_k(int32_t k)
{
    return (double)(64 + (k & 63)) * ldexp(1.0, (k >> 6) - 14);
}

/* Largest admissible k for a row length: |v| stays below 2^21 so that every coordinate
 * is exact in fp32 and its token input stays below 2^22. */
int32_t or_k_max(int64_t cols)
{
    double lim = ldexp(1.0, 20) / (sqrt((double)cols) + 1.0);
    int32_t k = NQ - 1;
    while (k > 0 && or_q_of_k(k) > lim)
        k--;
    return k;
}

/* ---------------------------------- lattice quantizer -------------------------------- */
/* Nearest point of D8 = {r in Z^8 : sum r even} (Conway & Sloane): round every
 * coordinate to the nearest integer (ties to even); if the sum is odd, move the
 * coordinate with the largest rounding error (lowest index on ties) to its other
 * neighbouring integer (upwards when that coordinate was already an integer). */
void or_d8_nearest(const double *y, double *r)
{
    long long sum = 0;
    for (int i = 0; i < 8; i++) {
        r[i] = nearbyint(y[i]);
        sum += (long long)r[i];
    }
    if (sum % 2 != 0) {
        int j = 0;
        double worst = -1.0;
        for (int i = 0; i < 8; i++) {
            double d = fabs(y[i] - r[i]);
            if (d > worst) {
                worst = d;
                j = i;
            }
        }
        if (y[j] < r[j])
            r[j] -= 1.0;
        else
            r[j] += 1.0;
    }
}

/* Nearest point of E8 = D8 u (D8 + 1/2): decode x in D8 and x - 1/2 in D8 (+1/2),
 * keep the closer (squared errors summed in coordinate order; a tie keeps the integer
 * coset).  Returns v = 2z so that both cosets are integers: all v_i even (integer
 * coset) or all odd, and sum v = 0 mod 4. */
void or_e8_nearest(const double *x, int32_t *v)
{
    double ya[8], yb[8], ra[8], rb[8], da = 0.0, db = 0.0;
    for (int i = 0; i < 8; i++) {
        ya[i] = x[i];
        yb[i] = x[i] - 0.5;
    }
    or_d8_nearest(ya, ra);
    or_d8_nearest(yb, rb);
    for (int i = 0; i < 8; i++) {
        double e = ya[i] - ra[i];
        da += e * e;
    }
    for (int i = 0; i < 8; i++) {
        double e = yb[i] - rb[i];
        db += e * e;
    }
    if (db < da)
        for (int i = 0; i < 8; i++)
            v[i] = 2 * (int32_t)rb[i] + 1;
    else
        for (int i = 0; i < 8; i++)
            v[i] = 2 * (int32_t)ra[i];
}

void or_e8_nearest_batch(const double *x, int64_t nblocks, int32_t *v)
{
    for (int64_t b = 0; b < nblocks; b++)
        or_e8_nearest(x + 8 * b, v + 8 * b);
}

/* ---------------------------------- symbols ------------------------------------------ */
uint32_t or_zigzag(int32_t y) { return y >= 0 ? 2u * (uint32_t)y : 2u * (uint32_t)(-(int64_t)y) - 1u; }

int32_t or_unzigzag(uint32_t u) { return (u & 1u) ? -(int32_t)((u + 1u) / 2u) : (int32_t)(u / 2u); }

/* a mod b in [0, b) for b > 0 (C's % truncates toward zero) */
static int32_t mod_floor(int32_t a, int32_t b)
{
    int32_t r = a % b;
    return r < 0 ? r + b : r;
}

/* Conditional model (reading of [ABS] "conditional probability model of lattice
 * coordinates"): the coordinates of one block v = 2z are coded in order 0..7.  The coset is
 * c = v0 mod 2 and y_i = (v_i - c) / 2; p = (y_0 + ... + y_6) mod 2.
 *   coordinate 0: context 0, value 4 zigzag(a0) + r0 with v0 = 4 a0 + r0, r0 in [0, 4):
 *     its two low bits are the coset and the parity of y_0.
 *   coordinates 1..6: context 1 + c, value 2 zigzag(a) + b with y_i = 2 a + b, b in {0, 1}:
 *     its low bit is the parity of y_i.
 *   coordinate 7: context 3 + 2c + p.  E8 forces y_7 = p (mod 2), so the value is
 *     zigzag((y_7 - p) / 2).
 * The low bits named here are kept by every token (or_tokenize), so the contexts of a block
 * follow from its tokens alone. */
void or_block_symbols(const int32_t *v, uint32_t *ctx, uint32_t *s)
{
    int32_t c = mod_floor(v[0], 2);
    int32_t y[8], p = 0;
    for (int i = 0; i < 8; i++)
        y[i] = (v[i] - c) / 2; /* exact: v_i - c is even */
    for (int i = 0; i < 7; i++)
        p = mod_floor(p + y[i], 2);
    int32_t r0 = mod_floor(v[0], 4);
    ctx[0] = 0;
    s[0] = 4u * or_zigzag((v[0] - r0) / 4) + (uint32_t)r0;
    for (int i = 1; i < 7; i++) {
        int32_t b = mod_floor(y[i], 2);
        ctx[i] = 1u + (uint32_t)c;
        s[i] = 2u * or_zigzag((y[i] - b) / 2) + (uint32_t)b;
    }
    ctx[7] = 3u + 2u * (uint32_t)c + (uint32_t)p;
    s[7] = or_zigzag((y[7] - p) / 2);
}

/* Inverse of or_block_symbols for one block, coordinate by coordinate in coding order:
 * returns v and the context of every coordinate. */
void or_block_values(const uint32_t *s, int32_t *v, uint32_t *ctx)
{
    int32_t r0 = (int32_t)(s[0] % 4u);
    v[0] = 4 * or_unzigzag(s[0] / 4u) + r0;
    int32_t c = mod_floor(v[0], 2);
    int32_t p = mod_floor((v[0] - c) / 2, 2);
    ctx[0] = 0;
    for (int i = 1; i < 7; i++) {
        int32_t y = 2 * or_unzigzag(s[i] / 2u) + (int32_t)(s[i] % 2u);
        v[i] = 2 * y + c;
        p = mod_floor(p + y, 2);
        ctx[i] = 1u + (uint32_t)c;
    }
    int32_t y7 = 2 * or_unzigzag(s[7]) + p;
    v[7] = 2 * y7 + c;
    ctx[7] = 3u + 2u * (uint32_t)c + (uint32_t)p;
}

static uint32_t floor_log2(uint32_t u)
{
    uint32_t n = 0;
    while ((u >> (n + 1)) != 0)
        n++;
    return n;
}

/* Token binarization ("hybrid integer", with low bits kept): with split m, h = 2 and `low`
 * kept bits (m >= h + low), a value s < 2^m is its own token.  Otherwise, with
 * n = floor(log2 s), the token carries n, the h bits below the leading one and the `low`
 * lowest bits of s; the n - h - low bits in between travel as raw extra bits. */
void or_tokenize(uint32_t s, int32_t m, int32_t low, uint32_t *tok, uint32_t *nbits, uint32_t *extra)
{
    if (s < (1u << m)) {
        *tok = s;
        *nbits = 0;
        *extra = 0;
        return;
    }
    uint32_t n = floor_log2(s);
    uint32_t top = (s >> (n - H_BITS)) & ((1u << H_BITS) - 1u);
    uint32_t lo = s & ((1u << low) - 1u);
    *nbits = n - H_BITS - (uint32_t)low;
    *extra = (s >> low) & ((1u << *nbits) - 1u);
    *tok = (1u << m) + (((((n - (uint32_t)m) << H_BITS) | top) << low) | lo);
}

/* raw extra bits that follow a token */
static uint32_t token_extra_bits(uint32_t tok, int32_t m, int32_t low)
{
    if (tok < (1u << m))
        return 0;
    uint32_t n = (uint32_t)m + (((tok - (1u << m)) >> low) >> H_BITS);
    return n - H_BITS - (uint32_t)low;
}

uint32_t or_detokenize(uint32_t tok, int32_t m, int32_t low, uint32_t extra)
{
    if (tok < (1u << m))
        return tok;
    uint32_t d = tok - (1u << m);
    uint32_t lo = d & ((1u << low) - 1u), q = d >> low;
    uint32_t top = q & ((1u << H_BITS) - 1u);
    uint32_t n = (uint32_t)m + (q >> H_BITS);
    return (((1u << H_BITS) | top) << (n - H_BITS)) | (extra << low) | lo;
}

void or_detokenize_batch(const uint32_t *tok, int64_t n, int32_t m, int32_t low, const uint32_t *extra,
                         uint32_t *s)
{
    for (int64_t i = 0; i < n; i++)
        s[i] = or_detokenize(tok[i], m, low, extra[i]);
}

/* number of tokens a split can produce for values below 2^VALUE_BITS */
uint32_t or_alphabet_size(int32_t m, int32_t low)
{
    return (1u << m) + ((((uint32_t)(VALUE_BITS - m)) << H_BITS) << low);
}

void or_tokenize_batch(const uint32_t *s, int64_t n, int32_t m, int32_t low, uint32_t *tok, uint32_t *nbits,
                       uint32_t *extra)
{
    for (int64_t i = 0; i < n; i++)
        or_tokenize(s[i], m, low, tok + i, nbits + i, extra + i);
}

/* split of context c: the smallest m in [h + low, max split] with at least 99.9% of the
 * context's values below 2^m, else the largest split */
static int32_t choose_split(const uint64_t *bitlen_hist /* [VALUE_BITS + 1]: count by bit length */, int c)
{
    int32_t lo = H_BITS + CTX_LOW[c], hi = CTX_MAX_SPLIT[c];
    uint64_t n = 0;
    for (int i = 0; i <= VALUE_BITS; i++)
        n += bitlen_hist[i];
    if (n == 0)
        return lo;
    uint64_t below = 0;
    for (int32_t m = 0; m <= hi; m++) {
        below += bitlen_hist[m]; /* values with bit length m are below 2^m */
        if (m >= lo && below * 1000u >= n * 999u)
            return m;
    }
    return hi;
}

static int bit_length(uint32_t u)
{
    int n = 0;
    while (u) {
        n++;
        u >>= 1;
    }
    return n;
}

/* ---------------------------------- frequency tables --------------------------------- */
/* Counts -> frequencies summing to M (2^11 for token tables, 2^12 for pair tables) by largest
 * remainders: f_i = floor(c_i M / n);
 * the M - sum f_i leftover units go one each to the largest remainders (c_i M mod n),
 * lower index first on ties; then every seen token left at 0 is raised to 1 by taking a
 * unit from the currently largest frequency (lower index first on ties).  Every frequency
 * stays below M: a context with one seen token t gives it M - 1 and one unit to a phantom
 * token that never occurs (token 1 if t = 0, else token 0).  Returns the table length (last
 * token with f > 0, plus 1), or -1 for a single-token alphabet. */
static int32_t normalize_to(const uint64_t *counts, int32_t n, uint32_t M, uint32_t *f)
{
    uint64_t total = 0;
    int32_t len = 0;
    for (int32_t i = 0; i < n; i++) {
        total += counts[i];
        if (counts[i])
            len = i + 1;
        f[i] = 0;
    }
    if (total == 0)
        return 0;
    uint64_t *rem = (uint64_t *)calloc((size_t)n, sizeof(uint64_t));
    uint32_t sum = 0;
    for (int32_t i = 0; i < n; i++) {
        if (!counts[i])
            continue;
        /* c * M < 2^64 for any realistic count (c < 2^51) */
        f[i] = (uint32_t)((counts[i] * M) / total);
        rem[i] = (counts[i] * M) % total;
        sum += f[i];
    }
    uint32_t left = M - sum;
    unsigned char *given = (unsigned char *)calloc((size_t)n, 1);
    for (uint32_t r = 0; r < left; r++) {
        int32_t best = -1;
        for (int32_t i = 0; i < n; i++)
            if (counts[i] && !given[i] && (best < 0 || rem[i] > rem[best]))
                best = i;
        given[best] = 1;
        f[best] += 1;
    }
    for (int32_t i = 0; i < n; i++) {
        if (counts[i] && f[i] == 0) {
            int32_t big = 0;
            for (int32_t j = 1; j < n; j++)
                if (f[j] > f[big])
                    big = j;
            f[big] -= 1;
            f[i] = 1;
        }
    }
    free(rem);
    free(given);
    int32_t seen = 0, only = 0;
    for (int32_t i = 0; i < n; i++)
        if (counts[i]) {
            seen++;
            only = i;
        }
    if (seen == 1) {
        if (n < 2)
            return -1;
        int32_t phantom = only == 0 ? 1 : 0;
        f[only] = M - 1u;
        f[phantom] = 1;
        if (phantom + 1 > len)
            len = phantom + 1;
    }
    return len;
}

int32_t or_normalize_freqs(const uint64_t *counts, int32_t n, uint32_t *f)
{
    return normalize_to(counts, n, PROB_M, f);
}

int32_t or_normalize_freqs_to(const uint64_t *counts, int32_t n, int32_t bits, uint32_t *f)
{
    return normalize_to(counts, n, 1u << bits, f);
}

/* ---------------------------------- paired coding ----------------------------------- */
/* Pair table of a context with alphabet length A from the counts of its token pairs inside the
 * base (B * B of them, B = min(A, 40); index t_a B + t_b) and the count N of all its pairs: a pair
 * seen c > 0 times with c 2^16 < N, and every pair with a token outside the base, go to the
 * escape symbol B * B; the B * B + 1 counts are then normalised to 2^12.  rare[] (B * B) flags the
 * escaped pairs inside the base. */
void or_pair_table(const uint64_t *inside, uint32_t A, uint64_t N, uint32_t *freq, uint8_t *rare)
{
    uint32_t B = A < PAIR_BASE_MAX ? A : PAIR_BASE_MAX, n = B * B + 1;
    uint64_t *pc = (uint64_t *)calloc(n, sizeof(uint64_t));
    uint64_t in = 0;
    for (uint32_t q = 0; q + 1 < n; q++) {
        pc[q] = inside[q];
        in += inside[q];
        rare[q] = 0;
    }
    pc[n - 1] = N - in;
    for (uint32_t q = 0; q + 1 < n; q++)
        if (pc[q] && pc[q] * PAIR_RARE_SCALE < N) {
            rare[q] = 1;
            pc[n - 1] += pc[q];
            pc[q] = 0;
        }
    normalize_to(pc, (int32_t)n, PAIR_M, freq);
    free(pc);
}

/* pair base B of a context with token alphabet length A, and its table length (0: no table) */
static uint32_t pair_base(uint32_t A) { return A < PAIR_BASE_MAX ? A : PAIR_BASE_MAX; }
static uint32_t pair_table_len(uint32_t A) { return A ? pair_base(A) * pair_base(A) + 1u : 0u; }

/* raw bits of one token of an escaped pair: enough for A - 1 */
static uint32_t pair_raw_bits(uint32_t A) { return (uint32_t)bit_length(A > 1 ? A - 1 : 0); }

/* last token seen, plus one */
static uint32_t seen_len(const uint64_t *cnt, uint32_t n)
{
    uint32_t len = 0;
    for (uint32_t t = 0; t < n; t++)
        if (cnt[t])
            len = t + 1;
    return len;
}

/* The stream pairs coordinates 1..6 when it is asked to (OR_CODING_PAIRED) or, under automatic
 * coding, when it holds at least 2^17 blocks (the pair tables then cost under 1 % of a 4-bit
 * stream); in both cases only when every split keeps the coordinates' values in [-256, 255],
 * the alphabets of contexts 1 and 2 have at most 256 tokens and at most 1 / 2^12 of their tokens
 * (counted in cnt[1], cnt[2], of lengths n1, n2) lie at or beyond the base 40. */
static int pair_eligible(int32_t coding, int64_t nb, const int32_t *m, const uint64_t *cnt1, uint32_t n1,
                         const uint64_t *cnt2, uint32_t n2)
{
    if (coding == OR_CODING_SINGLE)
        return 0;
    for (int c = 0; c < NCTX; c++)
        if (m[c] > CTX_NARROW_SPLIT[c])
            return 0;
    const uint64_t *cnt[2] = {cnt1, cnt2};
    uint32_t n[2] = {n1, n2};
    for (int c = 0; c < 2; c++) {
        uint64_t all = 0, outside = 0;
        for (uint32_t t = 0; t < n[c]; t++) {
            all += cnt[c][t];
            if (t >= PAIR_BASE_MAX)
                outside += cnt[c][t];
        }
        if (seen_len(cnt[c], n[c]) > PAIR_MAX_ALPHABET || outside * PAIR_OUTSIDE_SCALE > all)
            return 0;
    }
    return coding == OR_CODING_PAIRED || nb >= PAIR_MIN_BLOCKS;
}

/* ---------------------------------- tiles -------------------------------------------- */
/* Reading of the tiles ([ABS]: each decodes without the others): a tile is 32 lanes x K blocks;
 * lane l of tile t owns blocks t*32K + 32k + l, k = 0..K-1.  K comes from the block count and
 * the target rate: the power of two at or below nb / 2^16 (at least 16, at most 256), which
 * keeps mid-sized matrices near 2048 tiles, then halved (down to 1) while the tile's expected
 * payload, 32 K blocks x 8 coordinates x target bits plus a tenth, exceeds 5952 bytes. */
uint32_t or_choose_blocks_per_lane(int64_t nb, double target)
{
    int64_t q = nb / 65536;
    uint32_t k = 16;
    while ((int64_t)k * 2 <= q && k < 256)
        k *= 2;
    while (k > 1 && 32.0 * (double)k * target * 1.1 > TILE_BUDGET)
        k /= 2;
    return k;
}

/* ---------------------------------- value preparation -------------------------------- */
static int is_code_container(int32_t c) { return c == ORD_INT8 || c == ORD_FP8E4M3; }

/* Per-row absmax INT8 / FP8 codes ([LIN]: the lossy coding applies to the codes themselves;
 * readings: INT8 uses the symmetric range [-127, 127]; an all-zero row gets scale 1). */
int or_prequant(const void *src, int32_t sdt, int64_t rows, int64_t cols, int32_t container, double *codes,
                float *scales)
{
    for (int64_t r = 0; r < rows; r++) {
        double amax = 0.0;
        for (int64_t j = 0; j < cols; j++) {
            double a = fabs(src_value(src, sdt, r * cols + j));
            if (a > amax)
                amax = a;
        }
        float s = 1.0f;
        if (amax > 0.0)
            s = (float)(amax / (container == ORD_INT8 ? 127.0 : 448.0));
        if (s == 0.0f) /* amax so small that the scale underflows */
            s = FLT_MIN;
        scales[r] = s;
        for (int64_t j = 0; j < cols; j++) {
            double w = src_value(src, sdt, r * cols + j);
            double c;
            if (amax == 0.0)
                c = 0.0;
            else if (container == ORD_INT8) {
                c = nearbyint(w / (double)s);
                if (c > 127.0)
                    c = 127.0;
                if (c < -127.0)
                    c = -127.0;
            } else {
                float t = (float)(w / (double)s);
                c = e4m3_value(or_e4m3_from_float(t));
            }
            codes[r * cols + j] = c;
        }
    }
    return OR_OK;
}

/* values the lattice stage sees: the source itself, or the INT8/FP8 codes */
static double *lattice_input(const void *src, int32_t sdt, int64_t rows, int64_t cols, int32_t container,
                             float *scales_out)
{
    double *w = (double *)malloc((size_t)(rows * cols) * sizeof(double));
    if (!w)
        return NULL;
    if (is_code_container(container)) {
        float *sc = scales_out ? scales_out : (float *)malloc((size_t)rows * sizeof(float));
        or_prequant(src, sdt, rows, cols, container, w, sc);
        if (!scales_out)
            free(sc);
    } else {
        for (int64_t i = 0; i < rows * cols; i++)
            w[i] = src_value(src, sdt, i);
    }
    return w;
}

/* "Row-normalized" (reading): each row is divided by its RMS s_r; the resolution q then
 * scales it, so the lattice input is x = w / (2 f_r) with f_r = s_r / (2q) rounded to
 * fp32 -- the same fp32 factor the decoder multiplies by.  s_r is the fp32 rounding of
 * sqrt(sum_j w_j^2 / C) with the sum taken left to right in double.  A row whose s_r is
 * 0 has f_r = 0 and all-zero lattice points; a factor that overflows fp32 is clamped to
 * FLT_MAX. */
static void row_rms(const double *w, int64_t rows, int64_t cols, float *s)
{
    for (int64_t r = 0; r < rows; r++) {
        double acc = 0.0;
        for (int64_t j = 0; j < cols; j++) {
            double a = w[r * cols + j];
            acc += a * a;
        }
        s[r] = (float)sqrt(acc / (double)cols);
    }
}

/* Rows whose length is not a multiple of 8 are zero-padded to the next multiple before
 * they are cut into E8 blocks (reading: the pages ask only for a non-empty 2-D tensor, so
 * the last block of a row holds the row's last cols % 8 values and zeros).  The padding
 * takes no part in the row statistics; its lattice coordinates are coded like any other
 * and dropped by the decoder.  Returns w itself when no padding is needed. */
static double *pad_rows(double *w, int64_t rows, int64_t cols)
{
    int64_t cp = (cols + 7) / 8 * 8;
    if (cp == cols)
        return w;
    double *wp = (double *)calloc((size_t)(rows * cp), sizeof(double));
    if (!wp)
        return NULL;
    for (int64_t r = 0; r < rows; r++)
        memcpy(wp + r * cp, w + r * cols, (size_t)cols * sizeof(double));
    return wp;
}

static float row_factor(float s, int32_t k)
{
    if (s == 0.0f)
        return 0.0f;
    float f = (float)((double)s / (2.0 * or_q_of_k(k)));
    if (isinf(f))
        f = FLT_MAX;
    return f;
}

static void quantize_block(const double *w, float f, int32_t *v)
{
    if (f == 0.0f) {
        for (int i = 0; i < 8; i++)
            v[i] = 0;
        return;
    }
    double x[8];
    for (int i = 0; i < 8; i++)
        x[i] = w[i] / (2.0 * (double)f);
    or_e8_nearest(x, v);
}

void or_row_factors(const void *src, int32_t sdt, int64_t rows, int64_t cols, int32_t container, int32_t k,
                    float *s_out, float *f_out)
{
    double *w = lattice_input(src, sdt, rows, cols, container, NULL);
    row_rms(w, rows, cols, s_out);
    for (int64_t r = 0; r < rows; r++)
        f_out[r] = row_factor(s_out[r], k);
    free(w);
}

int or_quantize(const void *src, int32_t sdt, int64_t rows, int64_t cols, int32_t container, int32_t k,
                int32_t *v)
{
    double *w = lattice_input(src, sdt, rows, cols, container, NULL);
    float *s = (float *)malloc((size_t)rows * sizeof(float));
    row_rms(w, rows, cols, s);
    double *wp = pad_rows(w, rows, cols);
    int64_t cb = (cols + 7) / 8;
    for (int64_t b = 0; b < rows * cb; b++) {
        int32_t vb[8];
        int64_t r = b / cb, c0 = 8 * (b % cb);
        quantize_block(wp + 8 * b, row_factor(s[r], k), vb);
        for (int i = 0; i < 8 && c0 + i < cols; i++)
            v[r * cols + c0 + i] = vb[i];
    }
    if (wp != w)
        free(wp);
    free(s);
    free(w);
    return OR_OK;
}

/* ---------------------------------- storage estimate --------------------------------- */
static size_t meta_bytes(int64_t rows, int32_t container, uint64_t total_tokens, uint32_t ntiles)
{
    size_t m = HEADER_BYTES + al16((size_t)rows * 4);
    if (is_code_container(container))
        m += al16((size_t)rows * 4);
    m += al16((size_t)total_tokens * 2);
    m += al16((size_t)(ntiles + 1) * 4);
    return m;
}

/* Sampled storage estimate ([ABS]: the resolution comes from storage estimated on a sample,
 * so the full stream is not encoded again and again).  Every S-th block (S = ceil(nb /
 * 65536)) is quantized at k; its symbols are tokenized with splits chosen on the sample,
 * and the payload is estimated as the sample's empirical conditional entropy of tokens
 * plus its raw extra bits, scaled by nb / n_sample.  Exact metadata is added, the table
 * length taken from the sample, plus 168 bytes per tile: a final state holds about 24 bits
 * that carry no payload (32 lanes x 3 bytes), the 32 word counts take 64 bytes and a tile
 * pads to 16 bytes (8 on average; the raw bits' last word is counted in that padding). */
static double estimate_bpp(const double *w, const float *s, int64_t rows, int64_t cols, int32_t container,
                           int32_t k, uint32_t K, int32_t coding)
{
    /* w: padded rows of 8 * ceil(cols / 8) values; the rate counts the cols true columns */
    int64_t cb = (cols + 7) / 8, nb = rows * cb;
    int64_t S = (nb + SAMPLE_TARGET - 1) / SAMPLE_TARGET;
    if (S < 1)
        S = 1;
    int64_t ns = (nb + S - 1) / S;
    uint32_t *ctx = (uint32_t *)malloc((size_t)ns * 8 * sizeof(uint32_t));
    uint32_t *u = (uint32_t *)malloc((size_t)ns * 8 * sizeof(uint32_t));
    uint64_t hist[NCTX][VALUE_BITS + 2];
    memset(hist, 0, sizeof hist);
    for (int64_t j = 0; j < ns; j++) {
        int64_t b = j * S;
        int32_t v[8];
        quantize_block(w + 8 * b, row_factor(s[b / cb], k), v);
        or_block_symbols(v, ctx + 8 * j, u + 8 * j);
        for (int i = 0; i < 8; i++)
            hist[ctx[8 * j + i]][bit_length(u[8 * j + i])]++;
    }
    int32_t m[NCTX];
    uint64_t *cnt[NCTX];
    for (int c = 0; c < NCTX; c++) {
        m[c] = choose_split(hist[c], c);
        cnt[c] = (uint64_t *)calloc(or_alphabet_size(m[c], CTX_LOW[c]), sizeof(uint64_t));
    }
    double extra = 0.0;
    for (int64_t i = 0; i < ns * 8; i++) {
        uint32_t t, nbits, ex;
        or_tokenize(u[i], m[ctx[i]], CTX_LOW[ctx[i]], &t, &nbits, &ex);
        cnt[ctx[i]][t]++;
        extra += (double)nbits;
    }
    double bits = 0.0;
    uint64_t total_tokens = 0;
    uint32_t lens[NCTX];
    for (int c = 0; c < NCTX; c++)
        lens[c] = seen_len(cnt[c], or_alphabet_size(m[c], CTX_LOW[c]));
    /* a paired stream stores pair tables for contexts 1 and 2; its payload is estimated by
     * the same token entropy */
    int paired = pair_eligible(coding, nb, m, cnt[1], or_alphabet_size(m[1], CTX_LOW[1]), cnt[2],
                               or_alphabet_size(m[2], CTX_LOW[2]));
    for (int c = 0; c < NCTX; c++) {
        uint64_t n = 0;
        for (uint32_t t = 0; t < or_alphabet_size(m[c], CTX_LOW[c]); t++)
            n += cnt[c][t];
        total_tokens += paired && (c == 1 || c == 2) ? pair_table_len(lens[c]) : lens[c];
        if (n == 0)
            continue;
        bits += (double)n * log2((double)n);
        for (uint32_t t = 0; t < or_alphabet_size(m[c], CTX_LOW[c]); t++)
            if (cnt[c][t])
                bits -= (double)cnt[c][t] * log2((double)cnt[c][t]);
    }
    bits += extra;
    uint32_t ntiles = (uint32_t)((nb + (int64_t)LANES * K - 1) / ((int64_t)LANES * K));
    double bytes = (double)meta_bytes(rows, container, total_tokens, ntiles) + 168.0 * (double)ntiles +
                   bits * ((double)nb / (double)ns) / 8.0;
    for (int c = 0; c < NCTX; c++)
        free(cnt[c]);
    free(ctx);
    free(u);
    return 8.0 * bytes / (double)(rows * cols);
}

double or_estimate_bpp(const void *src, int32_t sdt, int64_t rows, int64_t cols, int32_t container, int32_t k,
                       uint32_t K, int32_t coding)
{
    double *w = lattice_input(src, sdt, rows, cols, container, NULL);
    float *s = (float *)malloc((size_t)rows * sizeof(float));
    row_rms(w, rows, cols, s);
    double *wp = pad_rows(w, rows, cols);
    if (K == 0)
        K = or_choose_blocks_per_lane(rows * ((cols + 7) / 8), 4.0);
    double e = estimate_bpp(wp, s, rows, cols, container, k, K, coding);
    if (wp != w)
        free(wp);
    free(s);
    free(w);
    return e;
}

/* ---------------------------------- byte helpers ------------------------------------- */
static void put16(uint8_t *p, uint32_t v)
{
    p[0] = (uint8_t)v;
    p[1] = (uint8_t)(v >> 8);
}
static void put32(uint8_t *p, uint32_t v)
{
    for (int i = 0; i < 4; i++)
        p[i] = (uint8_t)(v >> (8 * i));
}
static void put64(uint8_t *p, uint64_t v)
{
    for (int i = 0; i < 8; i++)
        p[i] = (uint8_t)(v >> (8 * i));
}
static uint32_t get16(const uint8_t *p) { return (uint32_t)p[0] | ((uint32_t)p[1] << 8); }
static uint32_t get32(const uint8_t *p)
{
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t get64(const uint8_t *p) { return (uint64_t)get32(p) | ((uint64_t)get32(p + 4) << 32); }

/* ---------------------------------- tile encoder ------------------------------------- */
typedef struct {
    uint16_t f, cum;
    uint8_t bits; /* the symbol's table sums to 2^bits */
} event;

/* what the tile encoder needs of the stream's model */
typedef struct {
    int32_t m[NCTX];
    uint32_t *freq[NCTX], *cum[NCTX]; /* contexts 1 and 2 of a paired stream: the pair tables */
    int paired;
    uint32_t A[NCTX];   /* contexts 1 and 2 of a paired stream: token alphabet length */
    uint8_t *rare[NCTX]; /* contexts 1 and 2 of a paired stream: pair index -> coded as an escape */
} coder;

/* a token pair's symbol in a pair table of base B: its index, or the escape B * B */
static uint32_t pair_symbol(const coder *C, uint32_t c, uint32_t ta, uint32_t tb)
{
    uint32_t B = pair_base(C->A[c]);
    if (ta >= B || tb >= B || C->rare[c][ta * B + tb])
        return B * B;
    return ta * B + tb;
}

static void add_event(event *ev, size_t *ne, const coder *C, uint32_t c, uint32_t sym, uint32_t bits)
{
    ev[*ne].f = (uint16_t)C->freq[c][sym];
    ev[*ne].cum = (uint16_t)C->cum[c][sym];
    ev[*ne].bits = (uint8_t)bits;
    (*ne)++;
}

static void push_bits(uint8_t *raw, size_t *nraw, uint32_t v, uint32_t nbits)
{
    for (uint32_t j = 0; j < nbits; j++)
        raw[(*nraw)++] = (uint8_t)((v >> j) & 1u);
}

/* One block's rANS symbols (in decode order) and raw bits.  Single coding: the 8 tokens.
 * Paired coding: token 0, the pair symbols of coordinates (1,2), (3,4), (5,6), token 7; the raw
 * bits start with the two tokens of every escaped pair (first then second, each in
 * pair_raw_bits(A) bits).  Then, in both codings, the extra bits of coordinates 0..7. */
static void block_events(const coder *C, const uint32_t *ctx, const uint32_t *s, event *ev, size_t *ne,
                         uint8_t *raw, size_t *nraw)
{
    uint32_t tok[8], nbits[8], extra[8];
    for (int i = 0; i < 8; i++)
        or_tokenize(s[i], C->m[ctx[i]], CTX_LOW[ctx[i]], &tok[i], &nbits[i], &extra[i]);
    if (!C->paired) {
        for (int i = 0; i < 8; i++)
            add_event(ev, ne, C, ctx[i], tok[i], PROB_BITS);
    } else {
        uint32_t pc = ctx[1], A = C->A[pc], B = pair_base(A);
        int esc[3];
        add_event(ev, ne, C, ctx[0], tok[0], PROB_BITS);
        for (int j = 0; j < 3; j++) {
            uint32_t sym = pair_symbol(C, pc, tok[1 + 2 * j], tok[2 + 2 * j]);
            esc[j] = sym == B * B;
            add_event(ev, ne, C, pc, sym, PAIR_BITS);
        }
        add_event(ev, ne, C, ctx[7], tok[7], PROB_BITS);
        for (int j = 0; j < 3; j++)
            if (esc[j]) {
                push_bits(raw, nraw, tok[1 + 2 * j], pair_raw_bits(A));
                push_bits(raw, nraw, tok[2 + 2 * j], pair_raw_bits(A));
            }
    }
    for (int i = 0; i < 8; i++)
        push_bits(raw, nraw, extra[i], nbits[i]);
}

typedef struct {
    uint8_t *p;
    size_t n, cap;
} bytes;

static void bytes_put(bytes *b, const void *src, size_t n)
{
    if (b->n + n > b->cap) {
        size_t c = b->cap ? b->cap : 1024;
        while (c < b->n + n)
            c *= 2;
        b->p = (uint8_t *)realloc(b->p, c);
        b->cap = c;
    }
    memcpy(b->p + b->n, src, n);
    b->n += n;
}

/* Which block (row-major index row * cb + column block) lane l of tile t takes as its k-th.
 * Layout 0 (reading R15): tile t holds the 32K consecutive blocks from t * 32K, lane l the blocks
 * t*32K + 32k + l.  Layout 1 (reading R32, the block order of a consumer GEMM: one tile is one
 * operand tile of 128 output rows by 64 input columns; K = 32, rows a multiple of 128, columns a
 * multiple of 64): with KT = cb / 8 tiles across a row band, tile t covers rows
 * 128 (t / KT) .. +127 and column blocks 8 (t mod KT) .. +7, and lane l takes row 32 (k mod 4) + l
 * of the tile at column block k / 4, so that one step of the 32 lanes fills 32 consecutive rows of
 * one 8-column slice. */
static int64_t lane_block(int32_t layout, int64_t cb, int64_t t, int l, uint32_t K, uint32_t k)
{
    if (layout == 0)
        return t * (int64_t)LANES * K + (int64_t)k * LANES + l;
    int64_t kt = cb / 8;
    int64_t row = 128 * (t / kt) + 32 * (int64_t)(k % 4) + l;
    int64_t colb = 8 * (t % kt) + (int64_t)(k / 4);
    return row * cb + colb;
}

/* Decode order inside a tile (the rule both sides follow): the 32 lanes are independent
 * rANS coders, each with its own region of 16-bit words.  Lane l decodes its blocks
 * t*32K + 32k + l in order of k, and per block its rANS symbols in the order block_events
 * lists them; after every symbol the lane reads the next word from the front of its region if
 * its state fell below L.  After a block's symbols the lane takes the block's raw bits (in
 * block_events' order) from the back of its region: the region's last word holds the lane's
 * first 16 raw bits (least significant bit first), the word before it the next 16, and so on.
 * The encoder runs a lane's symbols in reverse, emitting words in reverse.  A tile stores the
 * 32 final encoder states (= initial decoder states, u32), the 32 region lengths in words
 * (u16), then the regions of lanes 0..31 one after another, zero padded to 16 bytes. */
static int encode_tile(const uint32_t *ctx, const uint32_t *s, int64_t nb, int64_t cb, int32_t layout, int64_t t,
                       uint32_t K, const coder *C, bytes *out)
{
    event *ev = (event *)malloc((size_t)K * 8 * sizeof(event));
    uint8_t *raw = (uint8_t *)malloc((size_t)K * (8 * VALUE_BITS + 48) + 16);
    uint16_t *words[LANES];
    size_t nw[LANES];
    uint32_t x[LANES];
    int rc = OR_OK;
    for (int l = 0; l < LANES; l++) {
        size_t ne = 0, nraw = 0;
        for (uint32_t k = 0; k < K; k++) {
            int64_t b = lane_block(layout, cb, t, l, K, k);
            if (b >= nb)
                break;
            block_events(C, ctx + 8 * b, s + 8 * b, ev, &ne, raw, &nraw);
        }
        size_t nrawords = (nraw + 15) / 16;
        words[l] = (uint16_t *)malloc((ne + nrawords + 1) * sizeof(uint16_t));
        nw[l] = 0;
        uint32_t st = STATE_L;
        uint16_t *rw = (uint16_t *)malloc((nrawords + 1) * sizeof(uint16_t));
        for (size_t j = 0; j < nrawords; j++) {
            uint32_t wd = 0;
            for (size_t q = 0; q < 16 && 16 * j + q < nraw; q++)
                wd |= (uint32_t)raw[16 * j + q] << q;
            rw[j] = (uint16_t)wd;
        }
        /* words[l] collects the region back to front: raw word 0 first, ..., then the rANS
         * words in the order the encoder emits them (the reverse of decode order) */
        for (size_t j = 0; j < nrawords; j++)
            words[l][nw[l]++] = rw[j];
        free(rw);
        for (size_t e = ne; e-- > 0;) {
            uint32_t f = ev[e].f, n = ev[e].bits;
            /* renormalise so that the encoded state stays below 2^32: x_max = (L >> n) << 16 * f */
            if ((uint64_t)st >= ((uint64_t)f << (32 - n))) {
                words[l][nw[l]++] = (uint16_t)(st & 0xffffu);
                st >>= 16;
            }
            st = ((st / f) << n) + (st % f) + ev[e].cum;
        }
        x[l] = st;
        if (nw[l] > 0xffffu)
            rc = OR_ERR_UNSUPPORTED;
    }
    uint8_t head[TILE_HEAD];
    for (int l = 0; l < LANES; l++) {
        put32(head + 4 * l, x[l]);
        put16(head + 4 * LANES + 2 * l, (uint32_t)nw[l]);
    }
    bytes_put(out, head, sizeof head);
    for (int l = 0; l < LANES; l++) {
        for (size_t i = 0; i < nw[l]; i++) {
            uint8_t w2[2];
            put16(w2, words[l][nw[l] - 1 - i]);
            bytes_put(out, w2, 2);
        }
        free(words[l]);
    }
    static const uint8_t zeros[16] = {0};
    size_t pad = al16(out->n) - out->n;
    bytes_put(out, zeros, pad);
    free(ev);
    free(raw);
    return rc;
}

/* ---------------------------------- full encode at one k ----------------------------- */
static int encode_at(const double *w, const float *s, const float *scales, int64_t rows, int64_t cols,
                     int32_t sdt, int32_t container, int32_t k, uint32_t K, int32_t coding, int32_t layout, uint8_t *out,
                     size_t cap, size_t *out_n)
{
    /* w: padded rows of 8 * ceil(cols / 8) values; the header keeps the true cols */
    int64_t cb = (cols + 7) / 8, nb = rows * cb;
    uint32_t *ctx = (uint32_t *)malloc((size_t)nb * 8 * sizeof(uint32_t));
    uint32_t *u = (uint32_t *)malloc((size_t)nb * 8 * sizeof(uint32_t));
    float *f = (float *)malloc((size_t)rows * sizeof(float));
    if (!ctx || !u || !f)
        return OR_ERR_INVALID_ARG;
    for (int64_t r = 0; r < rows; r++)
        f[r] = row_factor(s[r], k);
    uint64_t hist[NCTX][VALUE_BITS + 2];
    memset(hist, 0, sizeof hist);
    for (int64_t b = 0; b < nb; b++) {
        int32_t v[8];
        quantize_block(w + 8 * b, f[b / cb], v);
        or_block_symbols(v, ctx + 8 * b, u + 8 * b);
        for (int i = 0; i < 8; i++)
            hist[ctx[8 * b + i]][bit_length(u[8 * b + i])]++;
    }
    int32_t m[NCTX];
    uint32_t *freq[NCTX], *cum[NCTX];
    uint64_t *cnt[NCTX];
    uint32_t ntok[NCTX], alpha[NCTX];
    uint64_t total_tokens = 0;
    for (int c = 0; c < NCTX; c++) {
        m[c] = choose_split(hist[c], c);
        alpha[c] = or_alphabet_size(m[c], CTX_LOW[c]);
        cnt[c] = (uint64_t *)calloc(alpha[c], sizeof(uint64_t));
        freq[c] = (uint32_t *)calloc(alpha[c], sizeof(uint32_t));
        cum[c] = (uint32_t *)calloc(alpha[c], sizeof(uint32_t));
    }
    for (int64_t i = 0; i < nb * 8; i++) {
        uint32_t t, nbits, ex;
        or_tokenize(u[i], m[ctx[i]], CTX_LOW[ctx[i]], &t, &nbits, &ex);
        cnt[ctx[i]][t]++;
    }
    coder C;
    memset(&C, 0, sizeof C);
    uint32_t tablen[NCTX];
    C.paired = pair_eligible(coding, nb, m, cnt[1], alpha[1], cnt[2], alpha[2]);
    for (int c = 0; c < NCTX; c++) {
        C.m[c] = m[c];
        if (C.paired && (c == 1 || c == 2)) {
            /* pair table: counts of (t_a, t_b) over the whole tensor; pairs outside the base and
             * rare pairs escaped */
            uint32_t A = seen_len(cnt[c], alpha[c]), B = pair_base(A), n = pair_table_len(A);
            ntok[c] = A;
            tablen[c] = n;
            C.A[c] = A;
            C.rare[c] = (uint8_t *)calloc(n + 1, 1);
            free(freq[c]);
            free(cum[c]);
            freq[c] = (uint32_t *)calloc(n + 1, sizeof(uint32_t));
            cum[c] = (uint32_t *)calloc(n + 1, sizeof(uint32_t));
            uint64_t *pc = (uint64_t *)calloc(n + 1, sizeof(uint64_t));
            uint64_t N = 0;
            for (int64_t b = 0; b < nb; b++)
                if (ctx[8 * b + 1] == (uint32_t)c)
                    for (int j = 0; j < 3; j++) {
                        uint32_t ta, tb, nbits, ex;
                        or_tokenize(u[8 * b + 1 + 2 * j], m[c], CTX_LOW[c], &ta, &nbits, &ex);
                        or_tokenize(u[8 * b + 2 + 2 * j], m[c], CTX_LOW[c], &tb, &nbits, &ex);
                        if (ta < B && tb < B)
                            pc[ta * B + tb]++;
                        N++;
                    }
            if (n)
                or_pair_table(pc, A, N, freq[c], C.rare[c]);
            free(pc);
        } else {
            ntok[c] = (uint32_t)or_normalize_freqs(cnt[c], (int32_t)alpha[c], freq[c]);
            tablen[c] = ntok[c];
        }
        uint32_t a = 0;
        for (uint32_t t = 0; t < tablen[c]; t++) {
            cum[c][t] = a;
            a += freq[c][t];
        }
        C.freq[c] = freq[c];
        C.cum[c] = cum[c];
        total_tokens += tablen[c];
    }
    uint32_t T = (uint32_t)((nb + (int64_t)LANES * K - 1) / ((int64_t)LANES * K));
    bytes tiles = {0, 0, 0};
    uint32_t *dir = (uint32_t *)malloc(((size_t)T + 1) * sizeof(uint32_t));
    int trc = OR_OK;
    for (uint32_t t = 0; t < T; t++) {
        dir[t] = (uint32_t)(tiles.n / 16);
        if (encode_tile(ctx, u, nb, cb, layout, t, K, &C, &tiles) != OR_OK)
            trc = OR_ERR_UNSUPPORTED;
    }
    dir[T] = (uint32_t)(tiles.n / 16);

    size_t off_rowf = HEADER_BYTES;
    size_t off_scales = off_rowf + al16((size_t)rows * 4);
    size_t off_freq = off_scales + (is_code_container(container) ? al16((size_t)rows * 4) : 0);
    size_t off_dir = off_freq + al16((size_t)total_tokens * 2);
    size_t off_tiles = off_dir + al16(((size_t)T + 1) * 4);
    size_t total = off_tiles + tiles.n;
    int rc = trc;
    *out_n = total;
    if (rc != OR_OK) {
        /* a lane region longer than 65535 words (only reachable with a forced tile size) */
    } else if (total > cap || !out) {
        rc = OR_ERR_BUFFER_TOO_SMALL;
    } else {
        memset(out, 0, total);
        put32(out, MAGIC);
        put16(out + 4, VERSION);
        out[6] = (uint8_t)sdt;
        out[7] = (uint8_t)container;
        put64(out + 8, (uint64_t)rows);
        put64(out + 16, (uint64_t)cols);
        put32(out + 24, T);
        put32(out + 28, K);
        put16(out + 32, (uint32_t)k);
        out[34] = PROB_BITS;
        out[35] = NCTX;
        out[43] = (uint8_t)C.paired;
        out[58] = (uint8_t)layout;
        for (int c = 0; c < NCTX; c++) {
            out[36 + c] = (uint8_t)m[c];
            put16(out + 44 + 2 * c, ntok[c]);
        }
        for (int64_t r = 0; r < rows; r++) {
            uint32_t b;
            memcpy(&b, &f[r], 4);
            put32(out + off_rowf + 4 * r, b);
        }
        if (is_code_container(container))
            for (int64_t r = 0; r < rows; r++) {
                uint32_t b;
                memcpy(&b, &scales[r], 4);
                put32(out + off_scales + 4 * r, b);
            }
        size_t p = off_freq;
        for (int c = 0; c < NCTX; c++)
            for (uint32_t t = 0; t < tablen[c]; t++, p += 2)
                put16(out + p, freq[c][t]);
        for (uint32_t t = 0; t <= T; t++)
            put32(out + off_dir + 4 * t, dir[t]);
        memcpy(out + off_tiles, tiles.p, tiles.n);
    }
    for (int c = 0; c < NCTX; c++) {
        free(cnt[c]);
        free(freq[c]);
        free(cum[c]);
        free(C.rare[c]);
    }
    free(tiles.p);
    free(dir);
    free(f);
    free(u);
    free(ctx);
    return rc;
}

/* ---------------------------------- compress ----------------------------------------- */
int or_compress(const void *src, int32_t sdt, int64_t rows, int64_t cols, double target, int32_t container,
                uint32_t K, int32_t q_override, int32_t coding, uint8_t *out, size_t cap, size_t *out_n)
{
    return or_compress_layout(src, sdt, rows, cols, target, container, K, q_override, coding, 0, out, cap, out_n);
}

int or_compress_layout(const void *src, int32_t sdt, int64_t rows, int64_t cols, double target, int32_t container,
                       uint32_t K, int32_t q_override, int32_t coding, int32_t layout, uint8_t *out, size_t cap,
                       size_t *out_n)
{
    if (!src || !out_n || rows <= 0 || cols <= 0)
        return OR_ERR_INVALID_ARG;
    /* layout 1 (R32): GEMM operand tiles of 128 rows x 64 columns, 32 blocks per lane */
    if (layout < 0 || layout > 1)
        return OR_ERR_INVALID_ARG;
    if (layout == 1) {
        if (rows % 128 != 0 || cols % 64 != 0 || (K != 0 && K != 32))
            return OR_ERR_INVALID_ARG;
        K = 32;
    }
    if (sdt != ORD_BF16 && sdt != ORD_FP16 && sdt != ORD_FP32)
        return OR_ERR_UNSUPPORTED;
    if (container == 0)
        container = sdt;
    if (container < ORD_BF16 || container > ORD_FP8E4M3)
        return OR_ERR_INVALID_ARG;
    if (K > 4096 || coding < OR_CODING_AUTO || coding > OR_CODING_PAIRED)
        return OR_ERR_INVALID_ARG;
    for (int64_t i = 0; i < rows * cols; i++)
        if (!isfinite(src_value(src, sdt, i)))
            return OR_ERR_NONFINITE;
    if (!(target >= 0.001) || !(target <= 11.0) || (is_code_container(container) && !(target < 8.0)))
        return OR_ERR_TARGET_RANGE;
    float *scales = (float *)malloc((size_t)rows * sizeof(float));
    double *w = lattice_input(src, sdt, rows, cols, container, scales);
    float *s = (float *)malloc((size_t)rows * sizeof(float));
    row_rms(w, rows, cols, s);
    double *wp = pad_rows(w, rows, cols);
    int64_t nb = rows * ((cols + 7) / 8);
    if (K == 0)
        K = or_choose_blocks_per_lane(nb, target);
    int32_t kmax = or_k_max(cols);
    int32_t k;
    if (q_override >= 0) {
        k = q_override > kmax ? kmax : q_override;
    } else {
        double budget = 0.995 * target;
        int32_t lo = 0, hi = kmax;
        while (lo < hi) {
            int32_t mid = lo + (hi - lo + 1) / 2;
            if (estimate_bpp(wp, s, rows, cols, container, mid, K, coding) <= budget)
                lo = mid;
            else
                hi = mid - 1;
        }
        k = lo;
    }
    int rc;
    for (;;) {
        size_t n = 0;
        rc = encode_at(wp, s, scales, rows, cols, sdt, container, k, K, coding, layout, NULL, 0, &n);
        if (rc == OR_ERR_UNSUPPORTED)
            break;
        if (q_override >= 0 || 8.0 * (double)n <= target * (double)(rows * cols)) {
            rc = encode_at(wp, s, scales, rows, cols, sdt, container, k, K, coding, layout, out, cap, out_n);
            break;
        }
        if (k == 0) {
            *out_n = n;
            rc = OR_ERR_TARGET_UNREACHABLE;
            break;
        }
        k--;
    }
    if (wp != w)
        free(wp);
    free(s);
    free(w);
    free(scales);
    return rc;
}

/* ---------------------------------- parse -------------------------------------------- */
int or_parse(const uint8_t *p, size_t n, or_info *info)
{
    if (!p || !info || n < HEADER_BYTES)
        return OR_ERR_CORRUPT;
    if (get32(p) != MAGIC || get16(p + 4) != VERSION || p[34] != PROB_BITS || p[35] != NCTX)
        return OR_ERR_CORRUPT;
    memset(info, 0, sizeof *info);
    info->src_dtype = p[6];
    info->container_dtype = p[7];
    info->rows = (int64_t)get64(p + 8);
    info->cols = (int64_t)get64(p + 16);
    info->n_tiles = get32(p + 24);
    info->blocks_per_lane = get32(p + 28);
    info->q_index = (int32_t)get16(p + 32);
    if (info->src_dtype < ORD_BF16 || info->src_dtype > ORD_FP32 || info->container_dtype < ORD_BF16 ||
        info->container_dtype > ORD_FP8E4M3)
        return OR_ERR_CORRUPT;
    if (info->rows <= 0 || info->cols <= 0 || info->rows > ((int64_t)1 << 40) ||
        info->cols > ((int64_t)1 << 40) || info->blocks_per_lane == 0 || info->blocks_per_lane > 4096)
        return OR_ERR_CORRUPT;
    int64_t nb = info->rows * ((info->cols + 7) / 8); /* rows padded to a multiple of 8 */
    int64_t T = (nb + (int64_t)LANES * info->blocks_per_lane - 1) / ((int64_t)LANES * info->blocks_per_lane);
    if (T != (int64_t)info->n_tiles)
        return OR_ERR_CORRUPT;
    if (p[43] > 1)
        return OR_ERR_CORRUPT;
    info->paired = p[43];
    /* byte 58: the block order of the tiles (0 row-major lanes, 1 GEMM operand tiles) */
    if (p[58] > 1)
        return OR_ERR_CORRUPT;
    info->layout = p[58];
    if (info->layout == 1 && (info->rows % 128 != 0 || info->cols % 64 != 0 || info->blocks_per_lane != 32))
        return OR_ERR_CORRUPT;
    uint64_t total_tokens = 0;
    for (int c = 0; c < NCTX; c++) {
        info->split[c] = p[36 + c];
        info->ntok[c] = (uint16_t)get16(p + 44 + 2 * c);
        if (info->split[c] < H_BITS + CTX_LOW[c] || info->split[c] > CTX_MAX_SPLIT[c] ||
            info->ntok[c] > or_alphabet_size(info->split[c], CTX_LOW[c]))
            return OR_ERR_CORRUPT;
        if (info->paired && info->split[c] > CTX_NARROW_SPLIT[c])
            return OR_ERR_CORRUPT;
        if (info->paired && (c == 1 || c == 2)) {
            if (info->ntok[c] > PAIR_MAX_ALPHABET)
                return OR_ERR_CORRUPT;
            total_tokens += pair_table_len(info->ntok[c]);
        } else {
            total_tokens += info->ntok[c];
        }
    }
    info->off_rowf = HEADER_BYTES;
    info->off_scales = info->off_rowf + al16((size_t)info->rows * 4);
    info->off_freq = info->off_scales + (is_code_container(info->container_dtype) ? al16((size_t)info->rows * 4) : 0);
    info->off_dir = info->off_freq + al16((size_t)total_tokens * 2);
    info->off_tiles = info->off_dir + al16(((size_t)T + 1) * 4);
    if (info->off_tiles > n)
        return OR_ERR_CORRUPT;
    /* tables sum to M, every frequency below M (2^12 for pair tables) */
    size_t q = info->off_freq;
    for (int c = 0; c < NCTX; c++) {
        int pair = info->paired && (c == 1 || c == 2);
        uint32_t len = pair ? pair_table_len(info->ntok[c]) : info->ntok[c], M = pair ? PAIR_M : PROB_M;
        uint32_t sum = 0;
        for (uint32_t t = 0; t < len; t++, q += 2) {
            if (get16(p + q) >= M)
                return OR_ERR_CORRUPT;
            sum += get16(p + q);
        }
        if (len && sum != M)
            return OR_ERR_CORRUPT;
    }
    /* directory: starts at 0, each tile holds at least its states, ends at the blob end */
    const uint8_t *d = p + info->off_dir;
    if (get32(d) != 0)
        return OR_ERR_CORRUPT;
    for (int64_t t = 0; t < T; t++)
        if (get32(d + 4 * (t + 1)) < get32(d + 4 * t) + TILE_HEAD / 16)
            return OR_ERR_CORRUPT;
    if (info->off_tiles + 16 * (uint64_t)get32(d + 4 * T) != n)
        return OR_ERR_CORRUPT;
    info->storage_nbytes = n;
    info->header_nbytes = HEADER_BYTES;
    info->actual_bpp = 8.0 * (double)n / (double)(info->rows * info->cols);
    return OR_OK;
}

/* ---------------------------------- decode ------------------------------------------- */
typedef struct {
    or_info in;
    const uint8_t *p;
    uint16_t *slot_tok[NCTX]; /* slot -> symbol (0xffff: slot outside the table) */
    uint32_t *freq[NCTX], *cum[NCTX];
    uint32_t len[NCTX], bits[NCTX]; /* table length; the table sums to 2^bits */
    const uint8_t *rowf;
    int32_t out_dtype; /* the container's dtype unless a float output dtype is asked for */
} dec_ctx;

static int dec_open(dec_ctx *D, const uint8_t *p, size_t n)
{
    int rc = or_parse(p, n, &D->in);
    if (rc)
        return rc;
    D->p = p;
    D->rowf = p + D->in.off_rowf;
    D->out_dtype = D->in.container_dtype;
    size_t q = D->in.off_freq;
    for (int c = 0; c < NCTX; c++) {
        int pair = D->in.paired && (c == 1 || c == 2);
        uint32_t nt = pair ? pair_table_len(D->in.ntok[c]) : D->in.ntok[c];
        uint32_t M = pair ? PAIR_M : PROB_M;
        D->len[c] = nt;
        D->bits[c] = pair ? PAIR_BITS : PROB_BITS;
        D->slot_tok[c] = (uint16_t *)malloc(M * sizeof(uint16_t));
        D->freq[c] = (uint32_t *)calloc(nt + 1, sizeof(uint32_t));
        D->cum[c] = (uint32_t *)calloc(nt + 1, sizeof(uint32_t));
        for (uint32_t s = 0; s < M; s++)
            D->slot_tok[c][s] = 0xffff;
        uint32_t a = 0;
        for (uint32_t t = 0; t < nt; t++, q += 2) {
            D->freq[c][t] = get16(p + q);
            D->cum[c][t] = a;
            for (uint32_t s = a; s < a + D->freq[c][t]; s++)
                D->slot_tok[c][s] = (uint16_t)t;
            a += D->freq[c][t];
        }
    }
    return OR_OK;
}

static void dec_close(dec_ctx *D)
{
    for (int c = 0; c < NCTX; c++) {
        free(D->slot_tok[c]);
        free(D->freq[c]);
        free(D->cum[c]);
    }
}

/* one lane's rANS step for a table symbol; returns the symbol */
static uint32_t dec_token(dec_ctx *D, uint32_t c, uint32_t *x, uint32_t *status, double *ideal)
{
    uint32_t n = D->bits[c];
    uint32_t slot = *x & ((1u << n) - 1u);
    uint32_t t = D->slot_tok[c][slot];
    if (t == 0xffff) {
        *status |= OR_DEC_BAD_TOKEN;
        return 0;
    }
    uint32_t f = D->freq[c][t];
    *x = f * (*x >> n) + slot - D->cum[c][t];
    if (ideal)
        *ideal += -log2((double)f / (double)(1u << n));
    return t;
}

typedef struct {
    uint64_t *tokcount[NCTX];
    double ideal, extra;
    uint64_t nsym;
} code_stats;

/* one lane's renormalisation: below L it reads the next word of its own stream */
static void dec_renorm(uint32_t *x, const uint8_t *wp, uint64_t nwords, uint64_t *pos, uint32_t *status)
{
    if (*x >= STATE_L)
        return;
    uint32_t wd = 0;
    if (*pos < nwords)
        wd = get16(wp + 2 * *pos);
    else
        *status |= OR_DEC_WORD_OVERRUN;
    (*pos)++;
    *x = (*x << 16) | wd;
}

/* a lane's raw extra bits: 16-bit words taken from the back of its region, each read least
 * significant bit first */
typedef struct {
    const uint8_t *region; /* the lane's first word */
    uint64_t len;          /* region length in words (as stored; may exceed the tile if damaged) */
    uint64_t avail;        /* words of the region inside the tile */
    uint64_t bit;          /* raw bits read so far */
} raw_reader;

static uint32_t raw_read(raw_reader *R, uint32_t nbits, uint32_t *status)
{
    uint32_t v = 0;
    for (uint32_t j = 0; j < nbits; j++, R->bit++) {
        uint64_t back = R->bit / 16; /* 0 = the region's last word */
        uint32_t bitv = 0;
        if (back < R->len && R->len - 1 - back < R->avail)
            bitv = (get16(R->region + 2 * (R->len - 1 - back)) >> (R->bit % 16)) & 1u;
        else
            *status |= OR_DEC_WORD_OVERRUN;
        v |= bitv << j;
    }
    return v;
}

/* Decodes tile t lane by lane in the order written down at encode_tile: each lane's tokens
 * from the front of its region, its raw extra bits from the back. */
static void decode_tile(dec_ctx *D, int64_t t, int32_t *vout, void *out, uint32_t *status, code_stats *cs)
{
    const or_info *I = &D->in;
    int64_t cb = (I->cols + 7) / 8, nb = I->rows * cb;
    uint32_t K = I->blocks_per_lane;
    const uint8_t *dir = D->p + I->off_dir;
    const uint8_t *tp = D->p + I->off_tiles + 16 * (uint64_t)get32(dir + 4 * t);
    uint64_t tile_bytes = 16 * (uint64_t)(get32(dir + 4 * (t + 1)) - get32(dir + 4 * t));
    uint64_t capacity = (tile_bytes - TILE_HEAD) / 2, start = 0;
    int esz = elt_size(D->out_dtype);
    for (int l = 0; l < LANES; l++) {
        uint32_t x = get32(tp + 4 * l);
        uint64_t len = get16(tp + 4 * LANES + 2 * l), pos = 0;
        const uint8_t *wp = tp + TILE_HEAD + 2 * start;
        uint64_t avail = start < capacity ? capacity - start : 0;
        if (avail > len)
            avail = len;
        if (start + len > capacity)
            *status |= OR_DEC_WORD_OVERRUN;
        start += len;
        raw_reader R = {wp, len, avail, 0};
        for (uint32_t k = 0; k < K; k++) {
            int64_t b = lane_block(I->layout, cb, t, l, K, k);
            if (b >= nb)
                break;
            uint32_t tok[8], ctx[8], sv[8];
            int32_t c = 0, p = 0;
            if (!I->paired) {
                for (int i = 0; i < 8; i++) {
                    ctx[i] = i == 0 ? 0u : i < 7 ? 1u + (uint32_t)c : 3u + 2u * (uint32_t)c + (uint32_t)p;
                    tok[i] = dec_token(D, ctx[i], &x, status, cs ? &cs->ideal : NULL);
                    dec_renorm(&x, wp, avail, &pos, status);
                    if (tok[i] >= I->ntok[ctx[i]])
                        *status |= OR_DEC_BAD_TOKEN;
                    if (cs) {
                        cs->tokcount[ctx[i]][tok[i] < D->len[ctx[i]] ? tok[i] : 0]++;
                        cs->nsym++;
                    }
                    /* the value's low bits do not depend on the extra bits (they are in the token) */
                    uint32_t lowbits = or_detokenize(tok[i], I->split[ctx[i]], CTX_LOW[ctx[i]], 0);
                    if (i == 0) {
                        c = (int32_t)(lowbits & 1u);
                        p = (int32_t)((lowbits >> 1) & 1u);
                    } else if (i < 7) {
                        p ^= (int32_t)(lowbits & 1u);
                    }
                }
            } else {
                /* paired: token 0, three pair symbols, the escaped pairs' tokens from the raw
                 * bits, token 7 */
                ctx[0] = 0;
                tok[0] = dec_token(D, 0, &x, status, cs ? &cs->ideal : NULL);
                dec_renorm(&x, wp, avail, &pos, status);
                if (tok[0] >= I->ntok[0])
                    *status |= OR_DEC_BAD_TOKEN;
                uint32_t low0 = or_detokenize(tok[0], I->split[0], CTX_LOW[0], 0);
                c = (int32_t)(low0 & 1u);
                p = (int32_t)((low0 >> 1) & 1u);
                uint32_t pc = 1u + (uint32_t)c, A = I->ntok[pc], B = pair_base(A), sym[3];
                for (int j = 0; j < 3; j++) {
                    sym[j] = dec_token(D, pc, &x, status, cs ? &cs->ideal : NULL);
                    dec_renorm(&x, wp, avail, &pos, status);
                    if (sym[j] >= D->len[pc])
                        *status |= OR_DEC_BAD_TOKEN;
                    if (cs) {
                        cs->tokcount[pc][sym[j] < D->len[pc] ? sym[j] : 0]++;
                        cs->nsym++;
                    }
                }
                for (int j = 0; j < 3; j++) {
                    uint32_t ta = 0, tb = 0;
                    if (A && sym[j] == B * B) {
                        ta = raw_read(&R, pair_raw_bits(A), status);
                        tb = raw_read(&R, pair_raw_bits(A), status);
                        if (ta >= A || tb >= A)
                            *status |= OR_DEC_BAD_TOKEN;
                        if (cs)
                            cs->extra += 2.0 * pair_raw_bits(A);
                    } else if (A) {
                        ta = sym[j] / B;
                        tb = sym[j] % B;
                    }
                    tok[1 + 2 * j] = ta;
                    tok[2 + 2 * j] = tb;
                }
                for (int i = 1; i < 7; i++) {
                    ctx[i] = pc;
                    p ^= (int32_t)(or_detokenize(tok[i], I->split[pc], CTX_LOW[pc], 0) & 1u);
                }
                ctx[7] = 3u + 2u * (uint32_t)c + (uint32_t)p;
                tok[7] = dec_token(D, ctx[7], &x, status, cs ? &cs->ideal : NULL);
                dec_renorm(&x, wp, avail, &pos, status);
                if (tok[7] >= I->ntok[ctx[7]])
                    *status |= OR_DEC_BAD_TOKEN;
                if (cs) {
                    cs->tokcount[0][tok[0] < D->len[0] ? tok[0] : 0]++;
                    cs->tokcount[ctx[7]][tok[7] < D->len[ctx[7]] ? tok[7] : 0]++;
                    cs->nsym += 2;
                }
            }
            for (int i = 0; i < 8; i++) {
                int32_t m = I->split[ctx[i]], low = CTX_LOW[ctx[i]];
                uint32_t nbits = token_extra_bits(tok[i], m, low);
                uint32_t extra = raw_read(&R, nbits, status);
                sv[i] = or_detokenize(tok[i], m, low, extra);
                if (cs)
                    cs->extra += nbits;
            }
            int32_t v[8];
            uint32_t ctx2[8];
            or_block_values(sv, v, ctx2);
            for (int i = 0; i < 8; i++)
                if (ctx2[i] != ctx[i])
                    *status |= OR_DEC_BAD_TOKEN;
            /* reconstruction: w = f_r * v in fp32, then the container conversion; a padded
             * row's last block keeps only its first cols % 8 values */
            int64_t r = b / cb, c0 = 8 * (b % cb);
            int n8 = I->cols - c0 < 8 ? (int)(I->cols - c0) : 8;
            uint32_t fb = get32(D->rowf + 4 * r);
            float fr;
            memcpy(&fr, &fb, 4);
            if (vout)
                memcpy(vout + r * I->cols + c0, v, (size_t)n8 * sizeof(int32_t));
            if (out) {
                float wv[8];
                for (int i = 0; i < 8; i++)
                    wv[i] = fr * (float)v[i];
                or_convert_batch(wv, n8, D->out_dtype, (uint8_t *)out + (size_t)(r * I->cols + c0) * (size_t)esz);
            }
        }
        if (x != STATE_L)
            *status |= OR_DEC_BAD_END;
        /* the front reads and the back reads cover the region exactly */
        uint64_t used = pos + (R.bit + 15) / 16;
        if (used != len)
            *status |= used > len ? OR_DEC_WORD_OVERRUN : OR_DEC_WORD_COUNT;
    }
    if (start > capacity || capacity - start >= 8)
        *status |= OR_DEC_WORD_COUNT;
}

int or_decode(const uint8_t *blob, size_t n, uint32_t t0, uint32_t t1, int32_t *v, void *out,
              uint32_t *status)
{
    return or_decode_as(blob, n, t0, t1, v, out, 0, status);
}

/* [API] CompressedTensor.to(dtype=...): the output dtype changes without recompression.
 * Reading: the fp32 weight f_r * v is rounded once into the requested dtype; a float
 * container (BF16 / FP16 / FP32) may decode to any of the three, a code container only to
 * its own dtype. */
int or_decode_as(const uint8_t *blob, size_t n, uint32_t t0, uint32_t t1, int32_t *v, void *out,
                 int32_t out_dtype, uint32_t *status)
{
    dec_ctx D;
    uint32_t st = 0;
    int rc = dec_open(&D, blob, n);
    if (rc)
        return rc;
    if (out_dtype) {
        int fo = out_dtype >= ORD_BF16 && out_dtype <= ORD_FP32;
        int fc = D.in.container_dtype >= ORD_BF16 && D.in.container_dtype <= ORD_FP32;
        if (out_dtype != D.in.container_dtype && !(fo && fc)) {
            dec_close(&D);
            return OR_ERR_INVALID_ARG;
        }
        D.out_dtype = out_dtype;
    }
    if (t1 > D.in.n_tiles)
        t1 = D.in.n_tiles;
    for (uint32_t t = t0; t < t1; t++)
        decode_tile(&D, t, v, out, &st, NULL);
    dec_close(&D);
    if (status)
        *status |= st;
    return OR_OK;
}

int or_code_stats(const uint8_t *blob, size_t n, double *ideal_bits, double *emp_entropy_bits, double *extra_bits,
                  uint64_t *n_symbols, uint64_t *payload_bytes)
{
    dec_ctx D;
    uint32_t st = 0;
    int rc = dec_open(&D, blob, n);
    if (rc)
        return rc;
    code_stats cs;
    memset(&cs, 0, sizeof cs);
    for (int c = 0; c < NCTX; c++)
        cs.tokcount[c] = (uint64_t *)calloc(D.len[c] + 1, sizeof(uint64_t));
    for (uint32_t t = 0; t < D.in.n_tiles; t++)
        decode_tile(&D, t, NULL, NULL, &st, &cs);
    double H = 0.0;
    for (int c = 0; c < NCTX; c++) {
        uint64_t tot = 0;
        for (uint32_t t = 0; t < D.len[c]; t++)
            tot += cs.tokcount[c][t];
        for (uint32_t t = 0; t < D.len[c]; t++)
            if (cs.tokcount[c][t])
                H += (double)cs.tokcount[c][t] * log2((double)tot / (double)cs.tokcount[c][t]);
        free(cs.tokcount[c]);
    }
    const uint8_t *dir = blob + D.in.off_dir;
    uint64_t pb = 0;
    for (uint32_t t = 0; t < D.in.n_tiles; t++)
        pb += 16 * (uint64_t)(get32(dir + 4 * (t + 1)) - get32(dir + 4 * t)) - TILE_HEAD;
    *ideal_bits = cs.ideal;
    *emp_entropy_bits = H;
    *extra_bits = cs.extra;
    *n_symbols = cs.nsym;
    *payload_bytes = pb;
    dec_close(&D);
    return st ? OR_ERR_CORRUPT : OR_OK;
}
