// Stream parser: ep_stream_info and ep_status_string.
//
// The CompressedTensor properties of the "EntroPack API reference" (shape, dtype,
// actual_bpp = 8 * storage_nbytes / numel, storage_nbytes with and without the header)
// read from a host copy of a format-v4 stream, which is validated before any decode.
#include <cstring>

#include "../../include/eptile.h"
#include "format.h"

namespace {

uint64_t rd(const uint8_t *p, int n) {
    uint64_t v = 0;
    for (int i = n - 1; i >= 0; --i) v = (v << 8) | p[i];
    return v;
}

}  // namespace

extern "C" int ep_stream_info(const void *blob, size_t nbytes, ep_info *info) {
    using namespace ep;
    if (!blob || !info) return EP_ERR_INVALID_ARG;
    const uint8_t *p = static_cast<const uint8_t *>(blob);
    if (nbytes < kHeaderBytes) return EP_ERR_CORRUPT;
    if (rd(p, 4) != kMagic || rd(p + 4, 2) != kVersion || p[34] != kProbBits || p[35] != kContexts)
        return EP_ERR_CORRUPT;
    ep_info I;
    std::memset(&I, 0, sizeof I);
    I.src_dtype = p[6];
    I.container_dtype = p[7];
    I.rows = int64_t(rd(p + 8, 8));
    I.cols = int64_t(rd(p + 16, 8));
    I.n_tiles = uint32_t(rd(p + 24, 4));
    I.blocks_per_lane = uint32_t(rd(p + 28, 4));
    I.q_index = int32_t(rd(p + 32, 2));
    if (I.src_dtype < EP_BF16 || I.src_dtype > EP_FP32 || I.container_dtype < EP_BF16 ||
        I.container_dtype > EP_FP8_E4M3)
        return EP_ERR_CORRUPT;
    if (I.rows <= 0 || I.cols <= 0 || I.rows >= (int64_t(1) << 40) || I.cols >= (int64_t(1) << 40) ||
        I.blocks_per_lane == 0 || I.blocks_per_lane > 4096 || I.q_index >= kNumQ)
        return EP_ERR_CORRUPT;
    // every product below is formed only once it is known to fit (rows and cols may each come
    // close to 2^40 in a damaged header)
    int64_t nb, elems, out_bytes;
    if (__builtin_mul_overflow(I.rows, (I.cols + 7) / 8, &nb) || __builtin_mul_overflow(I.rows, I.cols, &elems) ||
        __builtin_mul_overflow(elems, int64_t(elt_bytes(I.container_dtype)), &out_bytes))
        return EP_ERR_CORRUPT;
    // nb: rows zero-padded to whole E8 blocks
    int64_t per_tile = int64_t(kLanes) * I.blocks_per_lane;
    if ((nb + per_tile - 1) / per_tile != int64_t(I.n_tiles)) return EP_ERR_CORRUPT;
    if (p[43] > 1) return EP_ERR_CORRUPT;
    I.paired = p[43];
    // byte 58: the block order of the tiles (EP_LAYOUT_ROWS or EP_LAYOUT_GEMM)
    if (p[58] > 1) return EP_ERR_CORRUPT;
    I.layout = p[58];
    if (!layout_fits(int(I.layout), I.rows, I.cols, I.blocks_per_lane)) return EP_ERR_CORRUPT;
    uint64_t tokens = 0;
    uint32_t tablen[kContexts];
    for (int c = 0; c < kContexts; ++c) {
        I.split[c] = p[36 + c];
        I.ntok[c] = uint16_t(rd(p + 44 + 2 * c, 2));
        if (!split_valid(I.split[c], c) || I.ntok[c] > split_alphabet(I.split[c], kCtxLow[c])) return EP_ERR_CORRUPT;
        // a paired stream keeps every split in the narrow range and pairs alphabets of <= 256 tokens
        if (I.paired && I.split[c] > kCtxNarrowSplit[c]) return EP_ERR_CORRUPT;
        const bool pair = I.paired && (c == 1 || c == 2);
        if (pair && I.ntok[c] > kPairMaxAlphabet) return EP_ERR_CORRUPT;
        tablen[c] = pair ? pair_table_len(I.ntok[c]) : I.ntok[c];
        tokens += tablen[c];
    }
    Layout L = layout_for(I.rows, I.container_dtype, tokens, I.n_tiles);
    if (L.tiles > nbytes) return EP_ERR_CORRUPT;
    I.off_rowf = L.rowf;
    I.off_scales = L.scales;
    I.off_freq = L.freq;
    I.off_dir = L.dir;
    I.off_tiles = L.tiles;
    size_t q = L.freq;
    for (int c = 0; c < kContexts; ++c) {
        const uint32_t M = I.paired && (c == 1 || c == 2) ? kPairScale : kProbScale;
        uint32_t sum = 0;
        for (uint32_t t = 0; t < tablen[c]; ++t, q += 2) {
            uint32_t f = uint32_t(rd(p + q, 2));
            if (f >= M) return EP_ERR_CORRUPT;  // the decoder's table entry holds 11 (pairs: 12) bits
            sum += f;
        }
        if (tablen[c] && sum != M) return EP_ERR_CORRUPT;
    }
    const uint8_t *d = p + L.dir;
    uint64_t prev = rd(d, 4), largest = 0;
    if (prev != 0) return EP_ERR_CORRUPT;
    for (uint32_t t = 1; t <= I.n_tiles; ++t) {
        uint64_t cur = rd(d + 4 * t, 4);
        if (cur < prev + kTileHead / 16) return EP_ERR_CORRUPT;  // a tile holds at least its head
        if (cur - prev > largest) largest = cur - prev;
        prev = cur;
    }
    I.max_tile_nbytes = 16 * largest;
    if (L.tiles + 16 * prev != nbytes) return EP_ERR_CORRUPT;
    I.storage_nbytes = nbytes;
    I.header_nbytes = kHeaderBytes;
    I.actual_bpp = 8.0 * double(nbytes) / double(elems);
    I.out_nbytes = uint64_t(out_bytes);
    // the decoder's slot tables: 7 token tables, or 5 token tables, two pair tables of 8-byte
    // entries and the token fields of the escaped pairs
    I.workspace_nbytes = I.paired ? kPairedTableBytes : uint64_t(kContexts) * kProbScale * 4;
    *info = I;
    return EP_OK;
}

extern "C" const char *ep_status_string(int s) {
    switch (s) {
    case EP_OK: return "ok";
    case EP_ERR_INVALID_ARG: return "invalid argument";
    case EP_ERR_NONFINITE: return "tensor holds NaN or Inf";
    case EP_ERR_TARGET_RANGE: return "target_bpp outside the supported range";
    case EP_ERR_TARGET_UNREACHABLE: return "target_bpp below what the metadata alone needs";
    case EP_ERR_BUFFER_TOO_SMALL: return "output buffer too small";
    case EP_ERR_CORRUPT: return "stream fails validation";
    case EP_ERR_CUDA: return "CUDA runtime error";
    case EP_ERR_UNSUPPORTED: return "not supported by the stream format";
    default: return "unknown status";
    }
}
