// Stream format v4 constants and small helpers shared by the library's host encoder, the
// stream parser and the decode kernel.  The byte layout is fixed by the library (the pages
// give none): a 64-byte header, per-row factors, optional per-row code scales, per-context
// frequency tables, a tile directory and the tiles.
#pragma once
#include <cstddef>
#include <cstdint>

namespace ep {

constexpr uint32_t kMagic = 0x31545045u;  // "EPT1"
constexpr uint32_t kVersion = 4;
constexpr uint32_t kProbBits = 11;         // frequency precision: tables sum to 2^11, each entry below it
constexpr uint32_t kProbScale = 1u << kProbBits;
constexpr uint32_t kStateLow = 1u << 16;   // rANS state interval [2^16, 2^32), 16-bit words
constexpr int kLanes = 32;                 // interleaved states per tile = warp lanes
constexpr int kContexts = 7;
constexpr uint32_t kTopBits = 2;           // bits below the leading one carried by an escape token
constexpr uint32_t kValueBits = 22;        // every coded value is below 2^22
// low bits of the value kept in every token, and the largest split, per context: coordinate 0
// keeps v0 mod 4 (coset, parity of y0), coordinates 1..6 the parity of y_i, coordinate 7 none.
// At the largest splits a direct token decodes to v0 in [-256, 255] (coordinate 0) or to
// y = (v - c) / 2 in [-256, 255] (coordinates 1..7); up to the narrow splits below, v itself
// stays in [-256, 255].
constexpr uint32_t kCtxLow[kContexts] = {2, 1, 1, 0, 0, 0, 0};
constexpr uint32_t kCtxMaxSplit[kContexts] = {9, 9, 9, 8, 8, 8, 8};
constexpr uint32_t kCtxNarrowSplit[kContexts] = {9, 8, 8, 7, 7, 7, 7};
constexpr uint32_t kMaxAlphabet = 720;     // (1 << 9) + ((22 - 9) << 2 << 2): the largest context alphabet
// Paired coding: coordinates (1,2), (3,4), (5,6) of a block as one symbol each.  With A the
// context's token alphabet length and B = min(A, 40), a pair of tokens both below B is index
// t_a B + t_b of a table of B^2 + 1 symbols summing to 2^12; the last symbol is an escape, taken
// by pairs with a token at or above B and by pairs seen fewer than N / 2^16 times (N: the
// context's pair count), whose tokens follow in the raw bits.  Contexts 1 and 2 are paired while
// their alphabets have at most 256 tokens and at most 1 / 2^12 of their tokens lie at or beyond
// the base 40.  Header byte 43 holds 1 for a paired stream.
constexpr uint32_t kPairBits = 12;
constexpr uint32_t kPairScale = 1u << kPairBits;
constexpr uint32_t kPairBaseMax = 40;
constexpr uint32_t kPairMaxAlphabet = 256;
constexpr uint64_t kPairOutsideScale = 4096;
constexpr uint32_t kPairMaxTable = kPairBaseMax * kPairBaseMax + 1;
constexpr uint32_t kPairTokFields = kPairMaxAlphabet;  // token fields per coset in the decoder's tables
constexpr int64_t kPairMinBlocks = int64_t(1) << 17;  // automatic coding pairs from this many blocks on
constexpr uint64_t kPairRareScale = 65536;            // a pair seen c times is escaped when c 2^16 < N
// the decoder's tables for a paired stream: token tables of contexts 0, 3..6 (2048 4-byte slots
// each), pair tables of contexts 1, 2 (4096 8-byte slots each), and 2 x 256 token fields
constexpr uint64_t kPairedTableBytes = 5ull * 2048 * 4 + 2ull * 4096 * 8 + 2ull * kPairTokFields * 4;
constexpr size_t kHeaderBytes = 64;
constexpr size_t kTileHead = 192;            // per tile: 32 initial states (u32) + 32 word counts (u16)
                                             // then the lanes' words, then the tile's raw extra bits
constexpr double kTileBudget = 5952.0;       // expected payload bytes per tile (6 KB staging buffer)
constexpr int kNumQ = 1280;                // resolution indices
constexpr int64_t kSampleBlocks = 65536;   // blocks sampled by the storage estimate
constexpr double kTileOverheadBytes = 168.0;  // per tile in the estimate
constexpr double kTargetMargin = 0.995;

inline size_t align16(size_t n) { return (n + 15) & ~size_t(15); }

#ifdef __CUDACC__
#define EP_HD __host__ __device__
#else
#define EP_HD
#endif

// Block order of the tiles (header byte 58).  kLayoutRows: lane l of tile t codes blocks
// t*32K + 32k + l.  kLayoutGemm: every tile is one operand tile of a consumer GEMM, 128 rows by 64
// columns (K = 32, rows a multiple of 128, columns a multiple of 64); with KT = cb / 8 tiles
// across a row band, tile t covers rows 128 (t / KT) .. +127 and column blocks 8 (t mod KT) .. +7,
// and lane l codes row 32 (k mod 4) + l of it at column block k / 4, so one step of the 32 lanes
// covers 32 consecutive rows of one 8-column slice.
constexpr int kLayoutRows = 0;
constexpr int kLayoutGemm = 1;
constexpr int64_t kGemmTileRows = 128;
constexpr int64_t kGemmTileCols = 64;

// row-major index (row * cb + column block) of lane l's k-th block in tile t
EP_HD inline int64_t lane_block(int layout, int64_t cb, int64_t t, int l, uint32_t K, uint32_t k) {
    if (layout == kLayoutRows) return t * int64_t(kLanes) * K + int64_t(k) * kLanes + l;
    const int64_t kt = cb / 8;
    return (kGemmTileRows * (t / kt) + 32 * int64_t(k % 4) + l) * cb + 8 * (t % kt) + int64_t(k / 4);
}

// whether a shape and tile size can take a layout
inline bool layout_fits(int layout, int64_t rows, int64_t cols, uint32_t K) {
    if (layout == kLayoutRows) return true;
    return layout == kLayoutGemm && rows % kGemmTileRows == 0 && cols % kGemmTileCols == 0 && K == 32;
}

// tokens a split can produce for values below 2^22
inline uint32_t split_alphabet(uint32_t m, uint32_t low) { return (1u << m) + (((kValueBits - m) << kTopBits) << low); }

inline bool split_valid(uint32_t m, int ctx) { return m >= kTopBits + kCtxLow[ctx] && m <= kCtxMaxSplit[ctx]; }

inline uint32_t pair_base(uint32_t A) { return A < kPairBaseMax ? A : kPairBaseMax; }
inline uint32_t pair_table_len(uint32_t A) { return A ? pair_base(A) * pair_base(A) + 1u : 0u; }

// raw bits of one token of an escaped pair: the bit length of A - 1
inline uint32_t pair_raw_bits(uint32_t A) {
    uint32_t v = A > 1 ? A - 1 : 0, n = 0;
    while (v) {
        ++n;
        v >>= 1;
    }
    return n;
}

inline int elt_bytes(int dt) { return dt == 3 ? 4 : (dt == 1 || dt == 2) ? 2 : 1; }

inline bool is_code_container(int dt) { return dt == 4 || dt == 5; }

struct Layout {
    size_t rowf, scales, freq, dir, tiles;
};

inline Layout layout_for(int64_t rows, int container, uint64_t total_tokens, uint64_t ntiles) {
    Layout L;
    L.rowf = kHeaderBytes;
    L.scales = L.rowf + align16(size_t(rows) * 4);
    L.freq = L.scales + (is_code_container(container) ? align16(size_t(rows) * 4) : 0);
    L.dir = L.freq + align16(size_t(total_tokens) * 2);
    L.tiles = L.dir + align16(size_t(ntiles + 1) * 4);
    return L;
}

// K (blocks per lane) from the block count and the target rate: the power of two at or below
// nb / 2^16 (at least 16, at most 256), halved while a tile's expected payload (32 K blocks x 8
// coordinates x target bits, plus a tenth) exceeds the staging budget.
inline uint32_t auto_blocks_per_lane(int64_t nb, double target_bpp) {
    int64_t want = nb >> 16;
    uint32_t k = 16;
    while (k < 256 && int64_t(k) * 2 <= want) k <<= 1;
    while (k > 1 && 32.0 * double(k) * target_bpp * 1.1 > kTileBudget) k >>= 1;
    return k;
}

}  // namespace ep
