/*
 * eptile -- lattice-rANS weight streams with a fused B200 (sm_100a) decode.
 *
 * C ABI of libeptile.so.  Plain pointers and sizes only; no exceptions cross it; every
 * call returns an ep_status (0 = EP_OK, negative = error).  The library never allocates
 * device memory and never synchronises a stream: the caller owns every buffer.
 *
 * Sources (EntroPack pages, by title and section):
 *   "EntroPack API reference" -- compress(tensor, config) -> CompressedTensor,
 *       decompress(compressed) -> tensor with the same shape and dtype, CompressedTensor
 *       actual_bpp = 8 * storage_nbytes / numel and storage_nbytes(include_header).
 *   "EntroPack: Fast and Accurate Entropy-Coded Weight Compression at Arbitrary Bitrates",
 *       Abstract -- row-normalized E8 lattice quantization, a conditional model of the
 *       lattice coordinates, resolution chosen by sampled storage estimates, entropy coding
 *       in tiles that decode on their own, fused GPU symbol decode and reconstruction,
 *       BF16 / FP16 / FP8 / INT8 containers.
 *   "EntroPack README", Configuration -- 0.001 <= target_bpp <= 11.
 *   "Compressed Linear usage", Combine compression with FP8 or INT8 computation -- lossy
 *       compression of FP8 / INT8 weight codes, 0.001 <= target_bpp < 8, per-row scales
 *       counted in storage.
 * The byte layout of the stream (format version 4) is this library's own: a 64-byte header,
 * per-row factors, per-row code scales (INT8 / FP8), frequency tables, a tile directory and the
 * tiles (32 lane states, 32 region lengths, the lanes' words and raw bits).
 *
 * Decoding a stream takes two calls: ep_prepare once per device copy of a stream (it turns
 * the stream's frequency tables into the decoder's slot tables, in a caller-owned workspace
 * of info.workspace_nbytes), then ep_decompress as often as the weights are needed.
 */
#ifndef EPTILE_H
#define EPTILE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* same type as cudaStream_t; NULL is the legacy default stream */
typedef struct CUstream_st *ep_stream_t;

/* element types: source tensors (BF16, FP16, FP32) and containers (the first five).
 * EP_LATTICE_I32 is an output form only: the decoded lattice points v = 2z as int32. */
enum ep_dtype { EP_BF16 = 1, EP_FP16 = 2, EP_FP32 = 3, EP_INT8 = 4, EP_FP8_E4M3 = 5, EP_LATTICE_I32 = 6 };

enum ep_status {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = -1,        /* null pointer, empty or non-2-D shape, bad dtype/config */
    EP_ERR_NONFINITE = -2,          /* NaN or Inf in the source ("finite values", API reference) */
    EP_ERR_TARGET_RANGE = -3,       /* target_bpp outside [0.001, 11], or >= 8 for INT8/FP8 codes */
    EP_ERR_TARGET_UNREACHABLE = -4, /* even the coarsest resolution (metadata alone) exceeds the target */
    EP_ERR_BUFFER_TOO_SMALL = -5,   /* out_cap too small; *out_nbytes holds the size needed */
    EP_ERR_CORRUPT = -6,            /* the stream fails validation */
    EP_ERR_CUDA = -7,               /* a CUDA runtime call failed (launch, attribute) */
    EP_ERR_UNSUPPORTED = -8         /* valid but outside the format: >= 2^31 blocks (rows x ceil(cols / 8)),
                                       a lane region beyond 65535 words with a forced tile size */
};

/* bits the decode kernel ORs into *d_status when a stream is damaged */
enum ep_decode_flags {
    EP_DEC_WORD_OVERRUN = 1u, /* a renormalisation read ran past the tile's words */
    EP_DEC_BAD_TOKEN = 2u,    /* frequency tables that do not sum to 2^11 (pair tables: 2^12) or
                                 hold an entry of that much or more (ep_prepare); an escaped pair's
                                 token beyond its alphabet; a token outside its table (oracle) */
    EP_DEC_BAD_END = 4u,      /* a lane's state did not return to 2^16 at the end of its tile */
    EP_DEC_WORD_COUNT = 8u,   /* the tile has unread words beyond its 16-byte padding */
    EP_DEC_BAD_TILE = 16u,    /* a tile directory entry points outside the tile section */
    EP_DEC_TIMEOUT = 32u      /* a staging copy into shared memory did not complete within the
                                 kernel's poll limit; the CTA's remaining tiles are skipped */
};

typedef struct {
    double target_bpp;        /* bits per weight, including all metadata ("actual_bpp", API ref.) */
    int32_t container_dtype;  /* 0 = the source dtype; EP_INT8 / EP_FP8_E4M3 = per-row absmax codes */
    uint32_t blocks_per_lane; /* tile size K (blocks per lane); 0 = chosen from the shape */
    int32_t q_index;          /* -1 = search the resolution; >= 0 = encode at this resolution index */
    int32_t n_threads;        /* host encoder threads; 0 = all hardware threads */
    int32_t coding;           /* EP_CODING_*: how coordinates 1..6 of a block are coded */
    int32_t layout;           /* EP_LAYOUT_*: the block order of the tiles */
} ep_config;

/* EP_LAYOUT_ROWS: lane l of tile t codes blocks t*32K + 32k + l (the tiles follow the rows).
 * EP_LAYOUT_GEMM: every tile is one operand tile of a consumer GEMM, 128 rows by 64 columns (32
 * blocks per lane; rows a multiple of 128, columns a multiple of 64): tile t covers rows
 * 128 (t / KT) .. +127 and columns 64 (t mod KT) .. +63 with KT = cols / 64, and lane l codes row
 * 32 (k mod 4) + l of it at columns 8 (k / 4) .. +7. */
enum ep_layout { EP_LAYOUT_ROWS = 0, EP_LAYOUT_GEMM = 1 };

/* EP_CODING_AUTO pairs coordinates (1,2), (3,4), (5,6) of every block into one symbol each
 * when the stream holds at least 2^17 blocks and the tokens of their contexts concentrate below
 * 40 (at most 1 / 2^12 of them beyond, alphabets of at most 256 tokens; about 4.5 bpp and below):
 * 5 table lookups per block instead of 8 in the decoder, for well under 1 % more bits at 4 bpp;
 * EP_CODING_SINGLE never pairs; EP_CODING_PAIRED pairs whenever the tokens allow, at any size. */
enum ep_coding { EP_CODING_AUTO = 0, EP_CODING_SINGLE = 1, EP_CODING_PAIRED = 2 };

typedef struct {
    int64_t rows, cols;
    int32_t src_dtype, container_dtype;
    uint64_t storage_nbytes;  /* total stream bytes = storage_nbytes(include_header=True) */
    uint64_t header_nbytes;   /* 64; storage_nbytes - header_nbytes = include_header=False */
    double actual_bpp;        /* 8 * storage_nbytes / (rows * cols) */
    int32_t q_index;          /* resolution index k: lattice scale q = (64 + k%64) * 2^(k/64 - 14) */
    uint32_t n_tiles, blocks_per_lane;
    uint8_t split[8];         /* per-context token split m (7 contexts) */
    uint16_t ntok[8];         /* per-context table length (paired contexts 1, 2: token alphabet length A;
                                 their pair tables hold B * B + 1 entries, B = min(A, 40)) */
    uint64_t off_rowf;        /* byte offsets of the sections inside the stream */
    uint64_t off_scales;      /* INT8/FP8: per-row dequantization scales (fp32), for a GEMM consumer */
    uint64_t off_freq, off_dir, off_tiles;
    uint64_t out_nbytes;      /* rows * cols * container element size */
    uint64_t max_tile_nbytes; /* largest tile in the stream (sizes the decoder's staging buffers) */
    uint64_t workspace_nbytes;/* device workspace ep_prepare fills and ep_decompress reads: 57344,
                                 108544 for a paired stream */
    uint32_t paired;          /* 1: coordinates 1..6 are coded as three pairs per block */
    uint32_t layout;          /* EP_LAYOUT_*: the block order of the tiles */
} ep_info;

/* Upper bound of the stream size for ep_compress_host: with a searched resolution the
 * stream never exceeds floor(target_bpp * rows * cols / 8); with a fixed q_index the bound
 * is loose (metadata + 5 bytes per weight).  Returns 0 for invalid arguments. */
size_t ep_compress_bound(int64_t rows, int64_t cols, const ep_config *cfg);

/* compress(tensor, config) of the API reference, on the host.
 *   src        host pointer, row-major rows x cols elements of src_dtype (BF16/FP16/FP32),
 *              read only.
 *   cfg        target_bpp etc. (see ep_config); not retained.
 *   out        host buffer of out_cap bytes that receives the stream; caller-owned.
 *   out_nbytes receives the stream size (also on EP_ERR_BUFFER_TOO_SMALL: the size needed).
 * Steps (Abstract): optional per-row INT8/FP8 code preparation, row normalisation, a
 * resolution search on sampled storage estimates, E8 nearest-point quantization, per-context
 * frequency tables, tile-wise interleaved rANS.  The result satisfies actual_bpp <=
 * target_bpp or the call fails with EP_ERR_TARGET_UNREACHABLE.  Deterministic: the bytes do
 * not depend on n_threads.  Thread-safe (no global state). */
int ep_compress_host(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, const ep_config *cfg,
                     void *out, size_t out_cap, size_t *out_nbytes);

/* Scratch bytes ep_compress_device needs for this shape and config (0 for invalid arguments):
 * about 9 bytes per weight (context and value of every coordinate, the INT8 / FP8 code matrix)
 * plus small tables; it does not depend on the container or the data. */
size_t ep_compress_device_scratch(int64_t rows, int64_t cols, const ep_config *cfg);

/* compress(tensor, config) of the API reference with the tensor in DEVICE memory: the same stream
 * as ep_compress_host, byte for byte (same steps, same decisions), with the work over elements,
 * blocks and lanes on the GPU (row statistics, E8 quantization, token histograms, one rANS coder
 * per lane) and the decisions taken from integer histograms on the host (splits, frequency tables,
 * the sampled estimate and its bisection over the resolution, tile offsets).
 *   d_src       device pointer, row-major rows x cols elements of src_dtype (BF16/FP16/FP32).
 *   cfg         as for ep_compress_host (n_threads unused).
 *   d_out       device buffer of out_cap bytes (16-byte aligned) that receives the stream;
 *               ep_compress_bound gives a sufficient capacity.
 *   out_nbytes  receives the stream size (also on EP_ERR_BUFFER_TOO_SMALL / UNREACHABLE).
 *   d_scratch   device buffer of at least ep_compress_device_scratch bytes, 256-byte aligned,
 *               caller-owned; its contents are not needed afterwards.
 *   stream      CUDA stream of every launch and copy.
 * Errors as ep_compress_host.  Synchronous: the call waits on `stream` at each decision (a few
 * dozen times during the resolution search) and returns when the stream is written.  The
 * library allocates nothing. */
int ep_compress_device(const void *d_src, int32_t src_dtype, int64_t rows, int64_t cols, const ep_config *cfg,
                       void *d_out, size_t out_cap, size_t *out_nbytes, void *d_scratch, size_t scratch_nbytes,
                       ep_stream_t stream);

/* CompressedTensor's properties (API reference) from a HOST copy of the stream.
 *   blob   host pointer to the first nbytes of the stream; nbytes must be the whole stream
 *          (the tile directory is checked against the stream end).
 *   info   filled on success.
 * Validates magic, version, shape, dtypes, the coding byte, table sums (each used context sums
 * to 2048; a paired stream's pair tables to 4096) and the tile directory; returns EP_ERR_CORRUPT
 * otherwise. */
int ep_stream_info(const void *blob, size_t nbytes, ep_info *info);

/* First half of decompress(compressed) (API reference): the decoder's tables for one device
 * copy of a stream.  Run it once when the stream lands on the device; every ep_decompress of
 * that copy then reuses the workspace.
 *   info        from ep_stream_info on a host copy of the same stream.
 *   d_blob      device pointer to the whole stream, 16-byte aligned.
 *   d_workspace device buffer of info->workspace_nbytes bytes, 16-byte aligned, caller-owned;
 *               overwritten with 7 slot tables of 2048 32-bit entries (one per context: the
 *               token's frequency, the slot's offset in the token, the escape flag and the
 *               decoded value of a direct token: the coordinate v, or, when a split of the
 *               stream is beyond the narrow range (8 for coordinates 1..6, 7 for coordinate 7),
 *               y = (v - c) / 2 for coordinates 1..7).  A paired stream's workspace holds the
 *               slot tables of contexts 0 and 3..6, one 4096-slot table of 64-bit entries per
 *               coset (frequency, slot offset and the two coordinates' values, or an escape
 *               mark) and 2 x 256 token values for escaped pairs.
 *   d_status    nullable device uint32; EP_DEC_BAD_TOKEN is ORed in when the device copy's
 *               frequency tables are damaged.
 * One small kernel launch on `stream`; asynchronous. */
int ep_prepare(const ep_info *info, const void *d_blob, void *d_workspace, uint32_t *d_status,
               ep_stream_t stream);

/* decompress(compressed) of the API reference: the fused decode on the GPU.
 *   info        from ep_stream_info on a host copy of the same stream.
 *   d_blob      device pointer to the whole stream (info->storage_nbytes bytes), 16-byte aligned.
 *   d_workspace the workspace ep_prepare filled for this stream (read only here).
 *   d_out       device pointer to rows * cols elements of out_dtype, row-major, 16-byte aligned.
 *   out_dtype   info->container_dtype (the reconstructed weights or codes); for a BF16, FP16 or
 *               FP32 container also either of the other two ("to(dtype=...)" of the API
 *               reference: the output dtype changes without recompression; the fp32 weight
 *               f_r * v is rounded once, to nearest even, into out_dtype); or EP_LATTICE_I32 for
 *               the decoded lattice points v = 2z (int32) before scaling.  INT8 / FP8 code
 *               containers decode to their own dtype only.  Anything else: EP_ERR_INVALID_ARG.
 *   d_status    nullable device pointer to one uint32; the kernel ORs EP_DEC_* bits into it
 *               when it meets a damaged tile (clear it before the call to read it per call).
 *   stream      CUDA stream of the launch.
 * One kernel launch (sm_100a): a persistent grid, one CTA per SM, that bulk-copies the slot
 * tables and each warp's tiles into shared memory (TMA, mbarrier completion); each warp decodes
 * whole tiles with its 32 lanes as independent rANS coders, rebuilds the E8 coset in
 * registers, scales by the row factor in fp32 and stores the container with coalesced vector
 * stores.  Asynchronous: errors of the launch itself are returned; stream damage goes to
 * d_status.  The library allocates nothing and keeps a per-device cache of the SM count
 * only. */
int ep_decompress(const ep_info *info, const void *d_blob, const void *d_workspace, void *d_out, int32_t out_dtype,
                  uint32_t *d_status, ep_stream_t stream);

/* A linear layer's forward with the weight decoded inside the GEMM ("EntroPack API reference",
 * CompressedLinear and CompressedFP8Linear / CompressedINT8Linear: the weight is reconstructed for
 * every forward call; here it never reaches global memory): Y = X W^T (+ bias) for a stream written
 * with EP_LAYOUT_GEMM and a BF16, INT8 or FP8 E4M3 container.
 *   BF16:       the fp32 sum of the BF16 products, plus the bias, rounded once to BF16.
 *   INT8 / FP8: W8A8, as "Compressed Linear usage", Combine compression with FP8 or INT8
 *               computation: the activations are quantized per token (scale s_x = amax / 127 or
 *               / 448, 1 for an all-zero row; codes x / s_x rounded to nearest even and clamped to
 *               [-127, 127], or clamped to [-448, 448] and rounded to E4M3), the codes multiplied
 *               (INT8: exact int32 sums; FP8: fp32 sums), then y = RNE_bf16(fp32(fp32(sum) s_x) s_w)
 *               with s_w the stream's row scale, and with a bias RNE_bf16(y + bias).
 *   info        from ep_stream_info; W is info->rows (N, output features) x info->cols (K).
 *   d_blob      the stream in device memory (16-byte aligned); d_tables the slot tables
 *               ep_prepare built from it.
 *   d_x         BF16 activations, m x K row-major (16-byte aligned), 1 <= m <= 128.
 *   d_bias      nullable BF16 bias of N elements.
 *   d_y         BF16 output, m x N row-major: the fp32 sum rounded once to nearest even.
 *   d_work      caller-owned device scratch of ep_linear_fused_workspace(info, m) bytes, 16-byte
 *               aligned: the partial sums of the K splits, one counter per band of 128 output
 *               features and, for INT8 / FP8, the activations' codes and scales.  It must be
 *               zero-filled before its first use; every call leaves the counters at zero again.
 *               One call at a time per scratch buffer.
 *   d_status    nullable device uint32: EP_DEC_* bits of stream damage.
 * One launch (INT8 / FP8: after one launch that quantizes X): the stream's tiles in ranges over about
 * one wave of CTAs.  Their warps bulk-copy stream tiles into shared memory and decode them
 * straight into operand slices (128 features x 32 bytes: 16 BF16 weights or 32 codes) beside the
 * matching slices of X; one warp issues tcgen05.mma (kind::f16, kind::i8 or kind::f8f6f4; M = 128
 * features, N = m padded to 16) into the accumulator of the tile's band in tensor memory, read out
 * with tcgen05.ld into partial sums; a band's last CTA adds its CTAs' sums in order, scales and adds
 * the bias.
 * Asynchronous; allocates nothing.  EP_ERR_INVALID_ARG for another layout, container or m out of
 * range, EP_ERR_UNSUPPORTED when a tile is too large for the shared memory of one decoding warp. */
size_t ep_linear_fused_workspace(const ep_info *info, int64_t m);

/* The launch ep_linear_fused would make for this stream and m on a GPU with `sms` multiprocessors,
 * computed on the host without touching a device (for tests and capacity planning): the grid (each
 * band's K tiles split into ranges, about one wave of CTAs, or all tiles spread evenly over one wave
 * when that gives each decoding warp fewer rounds of tiles, more CTAs when one would touch more
 * bands than tensor memory holds accumulators for; the most tiles and the most bands of 128 output
 * features one CTA holds), the decoding warps per CTA, the padded token
 * count, the tensor-memory columns (one accumulator per band a CTA touches), the shared-memory
 * layout (tables from offset 0, then the barriers, the per-warp stream-tile buffers, the per-warp
 * pairs of 4 KB W slices and the per-warp X buffers) and the scratch bytes.  EP_ERR_INVALID_ARG as
 * ep_linear_fused refuses the stream or m, EP_ERR_UNSUPPORTED when even one decoding warp's buffers
 * do not fit (*out is filled either way). */
typedef struct {
    uint32_t bands, ctas, tiles_per_cta, accumulators;
    uint32_t spread;  /* 1: tiles spread evenly over the CTAs; 0: each band's K tiles in `splits` ranges */
    uint32_t splits;
    uint32_t decoding_warps, threads, tokens_padded, tmem_columns;
    uint32_t tile_buffer_bytes, smem_tables_bytes, smem_barriers_offset, smem_tiles_offset, smem_slices_offset;
    uint32_t smem_x_offset, smem_x_bytes_per_warp;
    uint64_t smem_bytes, work_bytes;
} ep_linear_plan;
int ep_linear_fused_plan(const ep_info *info, int64_t m, int32_t sms, ep_linear_plan *out);
int ep_linear_fused(const ep_info *info, const void *d_blob, const void *d_tables, const void *d_x, int64_t m,
                    const void *d_bias, void *d_y, void *d_work, size_t work_nbytes, uint32_t *d_status,
                    ep_stream_t stream);

/* ep_prepare + ep_decompress for callers that cannot allocate device memory: a plugin inside an
 * inference engine that owns all device memory and forbids allocation in its forward path, or code
 * that must not trigger the device-wide synchronisation a cudaMalloc/cudaFree can cause.  No
 * counterpart in the EntroPack pages; it exists for such callers only.
 *   Arguments as ep_decompress, without a workspace: the slot tables go to one file-scope device
 *   array of 108,544 bytes (info->workspace_nbytes of every stream), which each GPU that loads the
 *   library keeps until the process exits.  A stream needing more returns EP_ERR_UNSUPPORTED.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current and keeps it for the life of the process; make that first call before
 *   any stream capture.  A device reset (cudaDeviceReset, or the primary context torn down and
 *   created again) reloads the module and invalidates the kept address: do not call this entry
 *   point again in a process after resetting a device it was called on.
 *   All calls on a device share the array and leave the last call's tables in it: calls that
 *   overlap on the GPU (different streams without ordering) race and may decode with another
 *   stream's tables.  Two launches (tables, decode) on `stream`; no allocation, no sync. */
int ep_decompress_noalloc(const ep_info *info, const void *d_blob, void *d_out, int32_t out_dtype,
                          uint32_t *d_status, ep_stream_t stream);

/* Device scratch that ep_decompress_host needs for this stream and output dtype: the device copy
 * of the stream, the slot tables and the output, each rounded up to 256 bytes.  0 for invalid
 * arguments (an output dtype the stream cannot decode to included). */
size_t ep_decompress_host_scratch(const ep_info *info, int32_t out_dtype);

/* decompress(compressed) for a stream and an output in HOST memory (the API reference returns the
 * tensor on the compressed tensor's device): one copy of the stream to the device, ep_prepare,
 * ep_decompress, one copy of the output back, all on `stream`.  Asynchronous: synchronise the
 * stream before reading h_out; pinned host buffers let the copies run without staging.
 *   info        from ep_stream_info on the same stream.
 *   h_blob      host pointer to the whole stream (info->storage_nbytes bytes).
 *   h_out       host pointer to rows * cols elements of out_dtype (as for ep_decompress).
 *   d_scratch   device buffer of at least ep_decompress_host_scratch bytes, 256-byte aligned,
 *               caller-owned.
 *   d_status    nullable device uint32 (as for ep_decompress).
 * Errors as ep_decompress; the library allocates nothing. */
int ep_decompress_host(const ep_info *info, const void *h_blob, void *h_out, int32_t out_dtype, void *d_scratch,
                       size_t scratch_nbytes, uint32_t *d_status, ep_stream_t stream);

/* ---------------------------------------------------------------- the Tile-ANS lossless scheme
 * "EntroPack README", Configuration (TileANSConfig: lossless compression for BF16, FP16, FP32,
 * FP8 and INT8 tensors, the ratio depending on the data) and "EntroPack API reference",
 * decompress (lossless schemes restore every input bit).  The pages give no format; this
 * library's (format version 1): each element's most significant byte (the sign and top exponent
 * bits of a float, the whole byte of an 8-bit type) is rANS-coded with one static 256-symbol
 * table of 12-bit frequencies, in the lattice stream's lane tiles (chunks of 8 elements, 32 or 16
 * chunks per lane); the element's other bytes are kept as they are in a raw plane. */

typedef struct {
    int32_t dtype;            /* EP_BF16, EP_FP16, EP_FP32, EP_INT8 or EP_FP8_E4M3 */
    uint32_t blocks_per_lane; /* chunks of 8 elements per lane; 0 = 32, or 16 below 1024 tiles */
    int32_t n_threads;        /* host encoder threads; 0 = all hardware threads */
    int32_t reserved;         /* 0 */
} ep_ans_config;

typedef struct {
    int64_t n_elems;
    int32_t dtype, ndim;
    int64_t shape[8];         /* ndim dims, product n_elems */
    uint64_t storage_nbytes;  /* total stream bytes */
    double ratio;             /* storage_nbytes / (n_elems * element size) */
    uint32_t n_tiles, blocks_per_lane;
    uint64_t off_freq, off_dir, off_raw, off_tiles;
    uint64_t out_nbytes;      /* n_elems * element size */
    uint64_t max_tile_nbytes; /* largest tile (sizes the decoder's staging buffers) */
    uint64_t workspace_nbytes;/* 16384: the decoder's 4096-slot table */
} ep_ans_info;

/* Size of the Tile-ANS stream of n elements of `dtype` is at most this (0 for invalid
 * arguments): the raw bytes, one byte per element for the coded symbols plus their
 * worst-case growth, tables and tile heads. */
size_t ep_ans_compress_bound(int64_t n_elems, int32_t dtype);

/* compress(tensor, TileANSConfig()) on the host.
 *   src        host pointer to n_elems elements of cfg->dtype (any bit patterns: NaN payloads,
 *              infinities, signed zeros and subnormals are kept), read only.
 *   ndim/shape the tensor's shape (1..8 dims, product n_elems), stored for decompress.
 *   out        host buffer of out_cap bytes, caller-owned; out_nbytes receives the size (also on
 *              EP_ERR_BUFFER_TOO_SMALL: the size needed).
 * Byte-identical to the oracle's compressor.  Errors: EP_ERR_INVALID_ARG (null, empty, bad
 * dtype or shape), EP_ERR_BUFFER_TOO_SMALL, EP_ERR_UNSUPPORTED (a lane region beyond 65535
 * words with a forced tile size). */
int ep_ans_compress_host(const void *src, int64_t n_elems, int32_t ndim, const int64_t *shape,
                         const ep_ans_config *cfg, void *out, size_t out_cap, size_t *out_nbytes);

/* Parses and validates a host copy of a Tile-ANS stream (header, tables, directory and total
 * length).  EP_ERR_CORRUPT when it fails. */
int ep_ans_stream_info(const void *blob, size_t nbytes, ep_ans_info *info);

/* The decoder's slot table (4096 x u32: frequency, symbol, slot offset) from the stream's
 * frequencies, into a caller-owned device workspace of info->workspace_nbytes, 16-byte aligned;
 * once per device copy of a stream.  Tables that do not sum to 2^12 set EP_DEC_BAD_TOKEN in
 * d_status (nullable).  One small launch on `stream`; asynchronous. */
int ep_ans_prepare(const ep_ans_info *info, const void *d_blob, void *d_workspace, uint32_t *d_status,
                   ep_stream_t stream);

/* decompress(compressed) of a Tile-ANS stream in device memory: every element bit for bit.
 *   d_blob      device copy of the whole stream (16-byte aligned), caller-owned.
 *   d_workspace the table ep_ans_prepare filled from this copy.
 *   d_out       device buffer of info->out_nbytes (16-byte aligned): the tensor, row-major.
 *   d_status    nullable device uint32: EP_DEC_* bits of stream damage.
 * One persistent launch (one CTA per SM): the table and each warp's tiles staged in shared
 * memory by bulk copies, 32 rANS lanes per tile, each lane merging its decoded top bytes with
 * the raw plane and storing whole chunks.  Asynchronous; allocates nothing. */
int ep_ans_decompress(const ep_ans_info *info, const void *d_blob, const void *d_workspace, void *d_out,
                      uint32_t *d_status, ep_stream_t stream);

/* static string for a status code */
const char *ep_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif
