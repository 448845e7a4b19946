/*
 * Oracle for the lattice-rANS tile stream -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded C99 restatement of what the EntroPack pages
 * say the lossy path computes ("EntroPack: Fast and Accurate Entropy-Coded
 * Weight Compression at Arbitrary Bitrates", Abstract): row-normalized E8
 * lattice quantization, a conditional probability model of the lattice
 * coordinates, a resolution picked from sampled storage estimates, entropy
 * coding in independently decodable tiles, and decode with numerical
 * reconstruction into a weight container.  Where the pages leave a step open
 * (stream layout, model, tile size, rANS parameters) this file follows the
 * readings stated beside each function.
 *
 * Only the test-suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load this library.  It shares no source with the product
 * library (include/ and the package's csrc/); the two meet only through the
 * byte format of the stream.
 *
 * Parity status: every function below is pinned by tests/test_oracle_*.py
 * (brute force, closed forms, exact round trips, library cross-checks);
 * none is "parity unpinned" except the rate/distortion estimate below 2 bpp,
 * which is reported only.
 */
#ifndef EP_ORACLE_H
#define EP_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* dtype codes as they appear in the stream header */
enum { ORD_BF16 = 1, ORD_FP16 = 2, ORD_FP32 = 3, ORD_INT8 = 4, ORD_FP8E4M3 = 5 };

/* status codes (same numeric meaning as the product library's) */
enum {
    OR_OK = 0,
    OR_ERR_INVALID_ARG = -1,
    OR_ERR_NONFINITE = -2,
    OR_ERR_TARGET_RANGE = -3,
    OR_ERR_TARGET_UNREACHABLE = -4,
    OR_ERR_BUFFER_TOO_SMALL = -5,
    OR_ERR_CORRUPT = -6,
    OR_ERR_UNSUPPORTED = -8
};

/* coding of coordinates 1..6 asked of the compressor: automatic, one token per coordinate,
 * or paired whenever the token alphabets allow it (any tensor size) */
enum { OR_CODING_AUTO = 0, OR_CODING_SINGLE = 1, OR_CODING_PAIRED = 2 };

/* decode status bits (stream damage found while decoding a tile) */
enum {
    OR_DEC_WORD_OVERRUN = 1u,   /* a renormalisation or raw-bit read past the tile's words */
    OR_DEC_BAD_TOKEN = 2u,      /* a slot that maps to no token / token outside the table */
    OR_DEC_BAD_END = 4u,        /* a lane's final state differs from L */
    OR_DEC_WORD_COUNT = 8u      /* words left unread beyond the 16-byte padding */
};

typedef struct {
    int64_t rows, cols;
    int32_t src_dtype, container_dtype;
    uint64_t storage_nbytes, header_nbytes;
    double actual_bpp;
    int32_t q_index;
    uint32_t n_tiles, blocks_per_lane;
    uint8_t split[7];
    uint16_t ntok[7];
    uint64_t off_rowf, off_scales, off_freq, off_dir, off_tiles;
    uint32_t paired; /* 1: coordinates 1..6 coded as three pairs */
    uint32_t layout; /* block order of the tiles: 0 lanes along rows, 1 GEMM operand tiles (128 x 64) */
} or_info;

/* ---- scalar pieces, exposed so that tests can pin them one by one ---- */
double or_q_of_k(int32_t k);
int32_t or_k_max(int64_t cols);
void or_d8_nearest(const double *y, double *r);
void or_e8_nearest(const double *x, int32_t *v);
void or_e8_nearest_batch(const double *x, int64_t nblocks, int32_t *v);
uint32_t or_zigzag(int32_t y);
int32_t or_unzigzag(uint32_t u);
/* one block's contexts and values in coding order, and the inverse */
void or_block_symbols(const int32_t *v, uint32_t *ctx, uint32_t *s);
void or_block_values(const uint32_t *s, int32_t *v, uint32_t *ctx);
/* hybrid-integer tokens with split m and `low` low bits kept in every token */
void or_tokenize(uint32_t s, int32_t m, int32_t low, uint32_t *tok, uint32_t *nbits, uint32_t *extra);
uint32_t or_detokenize(uint32_t tok, int32_t m, int32_t low, uint32_t extra);
uint32_t or_alphabet_size(int32_t m, int32_t low);
void or_detokenize_batch(const uint32_t *tok, int64_t n, int32_t m, int32_t low, const uint32_t *extra,
                         uint32_t *s);
void or_tokenize_batch(const uint32_t *s, int64_t n, int32_t m, int32_t low, uint32_t *tok, uint32_t *nbits,
                       uint32_t *extra);
int32_t or_normalize_freqs(const uint64_t *counts, int32_t n, uint32_t *freqs);
/* the same rule for tables summing to 2^bits */
int32_t or_normalize_freqs_to(const uint64_t *counts, int32_t n, int32_t bits, uint32_t *freqs);
/* paired coding: the pair table (B * B + 1 frequencies summing to 2^12, B = min(A, 40)) of a
 * context with alphabet length A from its pair counts inside the base (B * B) and its pair count
 * N; rare (B * B) flags the pairs coded as the escape */
void or_pair_table(const uint64_t *inside, uint32_t A, uint64_t N, uint32_t *freq, uint8_t *rare);
uint32_t or_choose_blocks_per_lane(int64_t nblocks, double target_bpp);
uint16_t or_bf16_from_float(float w);
uint16_t or_fp16_from_float(float w);
uint8_t or_e4m3_from_float(float w);
int8_t or_int8_from_float(float w);
void or_convert_batch(const float *w, int64_t n, int32_t dtype, void *out);

/* container preparation for INT8 / FP8 codes: codes as exact doubles + per-row scale */
int or_prequant(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, int32_t container,
                double *codes, float *scales);
/* row statistics: rms s_r and factor f_r at resolution index k */
void or_row_factors(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, int32_t container,
                    int32_t k, float *s_out, float *f_out);
/* lattice points v = 2z (int32, rows*cols) at resolution index k */
int or_quantize(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, int32_t container,
                int32_t k, int32_t *v);
/* sampled storage estimate (bits per weight) at resolution index k; blocks_per_lane 0 takes
 * the automatic tile size for a 4 bpp target */
double or_estimate_bpp(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, int32_t container,
                       int32_t k, uint32_t blocks_per_lane, int32_t coding);

/* ---- the stream ---- */
/* q_override >= 0 skips the search and encodes at that index; blocks_per_lane 0 = automatic;
 * coding: OR_CODING_* */
int or_compress(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, double target_bpp,
                int32_t container, uint32_t blocks_per_lane, int32_t q_override, int32_t coding,
                uint8_t *out, size_t cap, size_t *out_nbytes);
/* or_compress with the tiles' block order: layout 0 (lane l of tile t takes blocks t*32K + 32k + l)
 * or layout 1 (each tile one 128-row x 64-column operand tile of a consumer GEMM; K = 32, rows a
 * multiple of 128, columns a multiple of 64) */
int or_compress_layout(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, double target_bpp,
                       int32_t container, uint32_t blocks_per_lane, int32_t q_override, int32_t coding,
                       int32_t layout, uint8_t *out, size_t cap, size_t *out_nbytes);
int or_parse(const uint8_t *blob, size_t nbytes, or_info *info);
/* decodes tiles [t0, t1): lattice points into v (indexed by weight, rows*cols, nullable) and
 * container bytes into out (rows*cols elements, nullable); returns OR_OK or a negative error,
 * and ORs OR_DEC_* bits into *status */
int or_decode(const uint8_t *blob, size_t nbytes, uint32_t t0, uint32_t t1, int32_t *v, void *out,
              uint32_t *status);
/* or_decode with the output rounded into out_dtype (0: the container's dtype); a float
 * container decodes to BF16, FP16 or FP32, a code container to its own dtype only
 * (OR_ERR_INVALID_ARG otherwise) */
int or_decode_as(const uint8_t *blob, size_t nbytes, uint32_t t0, uint32_t t1, int32_t *v, void *out,
                 int32_t out_dtype, uint32_t *status);
/* coding statistics over the whole stream, from a decode */
int or_code_stats(const uint8_t *blob, size_t nbytes, double *ideal_bits, double *emp_entropy_bits,
                  double *extra_bits, uint64_t *n_symbols, uint64_t *payload_bytes);

/* ---- the Tile-ANS lossless stream (ep_tile_ans.c) ---- */
typedef struct {
    int64_t n;               /* elements */
    int32_t dtype, ndim;
    int64_t shape[8];
    uint32_t n_tiles, blocks_per_lane;
    uint64_t off_freq, off_dir, off_raw, off_tiles, storage_nbytes;
} ota_info;

/* the tile size (chunks of 8 elements per lane) chosen for a tensor of n_chunks chunks */
uint32_t ota_blocks_per_lane(int64_t n_chunks);
/* compresses n elements of dtype (shape of ndim <= 8 dims, product n); blocks_per_lane 0 =
 * automatic; OR_ERR_BUFFER_TOO_SMALL with *out_nbytes = the size needed when cap is short */
int ota_compress(const void *src, int32_t dtype, int64_t n, int32_t ndim, const int64_t *shape,
                 uint32_t blocks_per_lane, uint8_t *out, size_t cap, size_t *out_nbytes);
int ota_parse(const uint8_t *blob, size_t nbytes, ota_info *info);
/* decodes tiles [t0, t1) into out (the tensor's bytes); ORs OR_DEC_* bits into *status */
int ota_decode(const uint8_t *blob, size_t nbytes, uint32_t t0, uint32_t t1, void *out, uint32_t *status);

#ifdef __cplusplus
}
#endif
#endif
