/*
 * Oracle for the Tile-ANS lossless stream -- TEST INFRASTRUCTURE ONLY (see ep_oracle.h).
 *
 * "EntroPack README", Configuration, and "EntroPack API reference", compress: TileANSConfig is
 * a lossless scheme for BF16, FP16, FP32, FP8 and INT8 tensors whose compression ratio depends
 * on the data; decompress restores every input bit.  The pages give no format.  This file
 * restates the readings the library follows:
 *   R28  symbols: the most significant byte of each element (sign and top exponent bits of a
 *        float; the whole byte of an 8-bit type) is entropy coded; the element's other bytes
 *        are stored as they are, in element order (the "raw plane").
 *   R29  model: one static table of 256 symbol frequencies per tensor, summing to 2^12, every
 *        entry below 2^12, by the same largest-remainder rule as the lattice stream's tables
 *        (or_normalize_freqs_to; a lone symbol gets 4095 and a phantom symbol 1).
 *   R30  tiles: the elements form chunks of 8 (the last one padded with zero elements, whose
 *        symbols are counted and coded); lane l of tile t owns chunks t*32K + 32k + l,
 *        k = 0..K-1, and codes their 8 symbols in element order with the lattice stream's rANS
 *        (32-bit state, L = 2^16, 16-bit words read from the front of the lane's region, states
 *        and word counts in a 192-byte tile head).
 *   R31  K: 32 chunks per lane, or 16 when 32 would leave fewer than 1024 tiles (a tile head of
 *        196 bytes then costs at most 0.38 bits per element); a caller may set it.
 * Stream: 64-byte header | shape (8 x i64) | 256 x u16 frequencies | tile directory (u32 x
 * (T+1), 16-byte units from the tile section) | raw plane | tiles; sections 16-byte aligned.
 * Header: 'EPA1', u16 version 1, u8 dtype, u8 ndim, i64 n, u32 T, u32 K, u8 probability bits
 * (12), zero to 64 bytes.
 *
 * Pinned by tests/test_oracle_tile_ans.py: bit-exact round trips of every dtype (including
 * NaN payloads, infinities, signed zeros, subnormals and incompressible bytes), the code length
 * against the empirical entropy of the symbols, and the stated stream layout.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "ep_oracle.h"

#define TA_MAGIC 0x31415045u /* "EPA1" */
#define TA_VERSION 1
#define TA_PROB_BITS 12
#define TA_M (1u << TA_PROB_BITS)
#define TA_L (1u << 16)
#define TA_LANES 32
#define TA_CHUNK 8
#define TA_HEAD 192
#define TA_MAXDIM 8

static size_t al16(size_t n) { return (n + 15) & ~(size_t)15; }

static int elt_size(int32_t dt)
{
    switch (dt) {
    case ORD_BF16:
    case ORD_FP16:
        return 2;
    case ORD_FP32:
        return 4;
    case ORD_INT8:
    case ORD_FP8E4M3:
        return 1;
    default:
        return 0;
    }
}

static void put16(uint8_t *p, uint32_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
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

uint32_t ota_blocks_per_lane(int64_t n_chunks)
{
    /* 32 chunks per lane (tile heads cost 0.19 bits per element), or 16 when that leaves fewer
     * than 1024 tiles to spread over the GPU */
    return (n_chunks + 32 * 32 - 1) / (32 * 32) >= 1024 ? 32u : 16u;
}

/* the section offsets of a stream of n elements of size esz in T tiles */
static void layout(int64_t n, int esz, uint32_t T, size_t *freq, size_t *dir, size_t *raw, size_t *tiles)
{
    *freq = 64 + 8 * TA_MAXDIM;
    *dir = *freq + 256 * 2;
    *raw = *dir + al16((size_t)(T + 1) * 4);
    *tiles = *raw + al16((size_t)n * (size_t)(esz - 1));
}

/* symbol of chunk element j (zero past the end) */
static uint32_t symbol_of(const uint8_t *src, int64_t n, int esz, int64_t i)
{
    return i < n ? src[i * esz + (esz - 1)] : 0u;
}

int ota_compress(const void *srcv, int32_t dtype, int64_t n, int32_t ndim, const int64_t *shape, uint32_t K,
                 uint8_t *out, size_t cap, size_t *n_out)
{
    const uint8_t *src = (const uint8_t *)srcv;
    int esz = elt_size(dtype);
    if (!src || !n_out || esz == 0 || n <= 0 || ndim < 1 || ndim > TA_MAXDIM || !shape)
        return OR_ERR_INVALID_ARG;
    int64_t prod = 1;
    for (int d = 0; d < ndim; d++) {
        if (shape[d] <= 0)
            return OR_ERR_INVALID_ARG;
        prod *= shape[d];
    }
    if (prod != n)
        return OR_ERR_INVALID_ARG;
    int64_t nc = (n + TA_CHUNK - 1) / TA_CHUNK;
    if (K == 0)
        K = ota_blocks_per_lane(nc);
    int64_t per_tile = (int64_t)TA_LANES * K;
    uint32_t T = (uint32_t)((nc + per_tile - 1) / per_tile);

    /* symbol counts over all chunks (padding included) and the frequency table */
    uint64_t cnt[256];
    memset(cnt, 0, sizeof cnt);
    for (int64_t i = 0; i < nc * TA_CHUNK; i++)
        cnt[symbol_of(src, n, esz, i)]++;
    uint32_t f[256], cum[257];
    or_normalize_freqs_to(cnt, 256, TA_PROB_BITS, f);
    cum[0] = 0;
    for (int s = 0; s < 256; s++)
        cum[s + 1] = cum[s] + f[s];

    /* every lane's words, encoded in reverse decode order */
    size_t maxw = (size_t)K * TA_CHUNK + 4; /* at most one word per symbol, plus the flush */
    uint16_t *words = (uint16_t *)malloc((size_t)T * TA_LANES * maxw * sizeof(uint16_t));
    uint32_t *nw = (uint32_t *)calloc((size_t)T * TA_LANES, sizeof(uint32_t));
    uint32_t *state = (uint32_t *)malloc((size_t)T * TA_LANES * sizeof(uint32_t));
    uint64_t tiles_bytes = 0;
    uint32_t *toff = (uint32_t *)malloc((size_t)(T + 1) * sizeof(uint32_t));
    for (uint32_t t = 0; t < T; t++) {
        uint64_t tw = 0;
        for (int l = 0; l < TA_LANES; l++) {
            uint16_t *w = words + ((size_t)t * TA_LANES + l) * maxw;
            uint32_t m = 0, x = TA_L;
            for (int64_t k = (int64_t)K - 1; k >= 0; k--) {
                int64_t c = (int64_t)t * per_tile + k * TA_LANES + l;
                if (c >= nc)
                    continue;
                for (int j = TA_CHUNK - 1; j >= 0; j--) {
                    uint32_t s = symbol_of(src, n, esz, c * TA_CHUNK + j);
                    uint32_t fs = f[s];
                    if (x >= (fs << 20)) { /* keeps x in [2^16, 2^32) after the update */
                        w[m++] = (uint16_t)(x & 0xffffu);
                        x >>= 16;
                    }
                    x = ((x / fs) << TA_PROB_BITS) + (x % fs) + cum[s];
                }
            }
            /* the decoder reads the words in the opposite order */
            for (uint32_t a = 0, b = m; a + 1 < b; a++, b--) {
                uint16_t tmp = w[a];
                w[a] = w[b - 1];
                w[b - 1] = tmp;
            }
            nw[(size_t)t * TA_LANES + l] = m;
            state[(size_t)t * TA_LANES + l] = x;
            tw += m;
        }
        toff[t] = (uint32_t)(tiles_bytes / 16);
        tiles_bytes += al16(TA_HEAD + 2 * tw);
    }
    toff[T] = (uint32_t)(tiles_bytes / 16);

    size_t o_freq, o_dir, o_raw, o_tiles;
    layout(n, esz, T, &o_freq, &o_dir, &o_raw, &o_tiles);
    size_t total = o_tiles + (size_t)tiles_bytes;
    *n_out = total;
    int rc = OR_OK;
    if (!out || cap < total) {
        rc = OR_ERR_BUFFER_TOO_SMALL;
        goto cleanup;
    }
    memset(out, 0, total);
    put32(out, TA_MAGIC);
    put16(out + 4, TA_VERSION);
    out[6] = (uint8_t)dtype;
    out[7] = (uint8_t)ndim;
    put64(out + 8, (uint64_t)n);
    put32(out + 16, T);
    put32(out + 20, K);
    out[24] = TA_PROB_BITS;
    for (int d = 0; d < ndim; d++)
        put64(out + 64 + 8 * d, (uint64_t)shape[d]);
    for (int s = 0; s < 256; s++)
        put16(out + o_freq + 2 * s, f[s]);
    for (uint32_t t = 0; t <= T; t++)
        put32(out + o_dir + 4 * t, toff[t]);
    for (int64_t i = 0; i < n; i++)
        for (int j = 0; j < esz - 1; j++)
            out[o_raw + (size_t)i * (esz - 1) + j] = src[i * esz + j];
    for (uint32_t t = 0; t < T; t++) {
        uint8_t *tp = out + o_tiles + 16 * (size_t)toff[t];
        size_t pos = TA_HEAD;
        for (int l = 0; l < TA_LANES; l++) {
            put32(tp + 4 * l, state[(size_t)t * TA_LANES + l]);
            put16(tp + 128 + 2 * l, nw[(size_t)t * TA_LANES + l]);
            const uint16_t *w = words + ((size_t)t * TA_LANES + l) * maxw;
            for (uint32_t a = 0; a < nw[(size_t)t * TA_LANES + l]; a++, pos += 2)
                put16(tp + pos, w[a]);
        }
    }
cleanup:
    free(words);
    free(nw);
    free(state);
    free(toff);
    return rc;
}

int ota_parse(const uint8_t *p, size_t nbytes, ota_info *I)
{
    if (!p || !I || nbytes < 64 + 8 * TA_MAXDIM + 512)
        return OR_ERR_CORRUPT;
    memset(I, 0, sizeof *I);
    if (get32(p) != TA_MAGIC || get16(p + 4) != TA_VERSION || p[24] != TA_PROB_BITS)
        return OR_ERR_CORRUPT;
    I->dtype = p[6];
    I->ndim = p[7];
    I->n = (int64_t)get64(p + 8);
    I->n_tiles = get32(p + 16);
    I->blocks_per_lane = get32(p + 20);
    int esz = elt_size(I->dtype);
    if (esz == 0 || I->ndim < 1 || I->ndim > TA_MAXDIM || I->n <= 0 || I->n >= ((int64_t)1 << 40) ||
        I->blocks_per_lane < 1 || I->blocks_per_lane > 4096)
        return OR_ERR_CORRUPT;
    int64_t prod = 1;
    for (int d = 0; d < I->ndim; d++) {
        I->shape[d] = (int64_t)get64(p + 64 + 8 * d);
        if (I->shape[d] <= 0 || I->shape[d] > I->n)
            return OR_ERR_CORRUPT;
        prod *= I->shape[d];
        if (prod > I->n)
            return OR_ERR_CORRUPT;
    }
    if (prod != I->n)
        return OR_ERR_CORRUPT;
    int64_t nc = (I->n + TA_CHUNK - 1) / TA_CHUNK, per_tile = (int64_t)TA_LANES * I->blocks_per_lane;
    if ((nc + per_tile - 1) / per_tile != (int64_t)I->n_tiles)
        return OR_ERR_CORRUPT;
    size_t o_freq, o_dir, o_raw, o_tiles;
    layout(I->n, esz, I->n_tiles, &o_freq, &o_dir, &o_raw, &o_tiles);
    if (o_tiles > nbytes)
        return OR_ERR_CORRUPT;
    uint32_t sum = 0;
    for (int s = 0; s < 256; s++) {
        uint32_t fs = get16(p + o_freq + 2 * s);
        if (fs >= TA_M)
            return OR_ERR_CORRUPT;
        sum += fs;
    }
    if (sum != TA_M)
        return OR_ERR_CORRUPT;
    uint32_t prev = get32(p + o_dir);
    if (prev != 0)
        return OR_ERR_CORRUPT;
    for (uint32_t t = 1; t <= I->n_tiles; t++) {
        uint32_t cur = get32(p + o_dir + 4 * t);
        if (cur < prev + TA_HEAD / 16)
            return OR_ERR_CORRUPT;
        prev = cur;
    }
    if (o_tiles + 16 * (size_t)prev != nbytes)
        return OR_ERR_CORRUPT;
    I->off_freq = o_freq;
    I->off_dir = o_dir;
    I->off_raw = o_raw;
    I->off_tiles = o_tiles;
    I->storage_nbytes = nbytes;
    return OR_OK;
}

/* Decodes tiles [t0, t1) into out (n elements of the stream's dtype); damage found on the way
 * is ORed into *status with the OR_DEC_* bits. */
int ota_decode(const uint8_t *p, size_t nbytes, uint32_t t0, uint32_t t1, void *outv, uint32_t *status)
{
    ota_info I;
    int rc = ota_parse(p, nbytes, &I);
    if (rc)
        return rc;
    if (t1 > I.n_tiles || t0 > t1 || !outv)
        return OR_ERR_INVALID_ARG;
    uint8_t *out = (uint8_t *)outv;
    int esz = elt_size(I.dtype);
    uint32_t f[256], cum[257];
    cum[0] = 0;
    for (int s = 0; s < 256; s++) {
        f[s] = get16(p + I.off_freq + 2 * s);
        cum[s + 1] = cum[s] + f[s];
    }
    int64_t nc = (I.n + TA_CHUNK - 1) / TA_CHUNK, per_tile = (int64_t)TA_LANES * I.blocks_per_lane;
    uint32_t st = 0;
    for (uint32_t t = t0; t < t1; t++) {
        size_t beg = I.off_tiles + 16 * (size_t)get32(p + I.off_dir + 4 * t);
        size_t end = I.off_tiles + 16 * (size_t)get32(p + I.off_dir + 4 * (t + 1));
        const uint8_t *tp = p + beg;
        size_t capacity = (end - beg - TA_HEAD) / 2, start = 0;
        for (int l = 0; l < TA_LANES; l++) {
            uint32_t x = get32(tp + 4 * l), len = get16(tp + 128 + 2 * l);
            size_t pos = 0;
            for (uint32_t k = 0; k < I.blocks_per_lane; k++) {
                int64_t c = (int64_t)t * per_tile + (int64_t)k * TA_LANES + l;
                if (c >= nc)
                    break;
                for (int j = 0; j < TA_CHUNK; j++) {
                    uint32_t slot = x & (TA_M - 1u);
                    uint32_t s = 0;
                    while (s < 255 && cum[s + 1] <= slot)
                        s++;
                    if (f[s] == 0)
                        st |= OR_DEC_BAD_TOKEN;
                    x = f[s] * (x >> TA_PROB_BITS) + slot - cum[s];
                    if (x < TA_L) {
                        uint32_t w = 0;
                        if (pos < len && start + pos < capacity)
                            w = get16(tp + TA_HEAD + 2 * (start + pos));
                        else
                            st |= OR_DEC_WORD_OVERRUN;
                        pos++;
                        x = (x << 16) | w;
                    }
                    int64_t i = c * TA_CHUNK + j;
                    if (i < I.n) {
                        for (int b = 0; b < esz - 1; b++)
                            out[i * esz + b] = p[I.off_raw + (size_t)i * (esz - 1) + b];
                        out[i * esz + esz - 1] = (uint8_t)s;
                    }
                }
            }
            if (x != TA_L)
                st |= OR_DEC_BAD_END;
            if (pos != len)
                st |= pos > len ? OR_DEC_WORD_OVERRUN : OR_DEC_WORD_COUNT;
            start += len;
        }
        if (start > capacity || capacity - start >= 8)
            st |= OR_DEC_WORD_COUNT;
    }
    if (status)
        *status |= st;
    return OR_OK;
}
