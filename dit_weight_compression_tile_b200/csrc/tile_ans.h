// Tile-ANS stream format v1 (the lossless scheme): constants and layout shared by the library's
// host compressor, its parser and the decode kernel.  The pages ("EntroPack README",
// Configuration: TileANSConfig) name the scheme and its dtypes only; the layout is the library's:
//   64-byte header | shape (8 x i64) | 256 x u16 symbol frequencies (sum 2^12, each below it) |
//   tile directory (u32 x (T + 1), 16-byte units from the tile section) | raw plane | tiles,
// every section 16-byte aligned.  Each element's most significant byte is its symbol; its other
// bytes sit in the raw plane, element by element.  Elements form chunks of 8 (the last padded
// with zero elements, whose symbols are coded); lane l of tile t codes chunks t*32K + 32k + l with
// the lattice stream's rANS (32-bit state, L = 2^16, 16-bit words; a tile head of 32 states and 32
// word counts, then the lanes' word regions, zero padding to 16 bytes).
#pragma once
#include <cstddef>
#include <cstdint>

namespace ep {
namespace ta {

constexpr uint32_t kMagic = 0x31415045u;  // "EPA1"
constexpr uint32_t kVersion = 1;
constexpr uint32_t kProbBits = 12;
constexpr uint32_t kProbScale = 1u << kProbBits;
constexpr uint32_t kStateLow = 1u << 16;
constexpr int kLanes = 32;
constexpr int kChunk = 8;                // elements per chunk (one lane step)
constexpr size_t kHeaderBytes = 64;
constexpr int kMaxDims = 8;
constexpr size_t kTileHead = 192;        // 32 initial states (u32) + 32 word counts (u16)
constexpr size_t kTableBytes = size_t(kProbScale) * 4;  // the decoder's slot table

inline size_t align16(size_t n) { return (n + 15) & ~size_t(15); }

// bytes per element of the dtypes the scheme takes (BF16, FP16, FP32, INT8, FP8 E4M3); 0 otherwise
inline int elt_bytes(int dt) { return dt == 1 || dt == 2 ? 2 : dt == 3 ? 4 : dt == 4 || dt == 5 ? 1 : 0; }

struct Layout {
    size_t freq, dir, raw, tiles;
};

inline Layout layout_for(int64_t n, int esz, uint64_t ntiles) {
    Layout L;
    L.freq = kHeaderBytes + 8 * kMaxDims;
    L.dir = L.freq + 256 * 2;
    L.raw = L.dir + align16(size_t(ntiles + 1) * 4);
    L.tiles = L.raw + align16(size_t(n) * size_t(esz - 1));
    return L;
}

// chunks per lane: 32 (tile heads cost 0.19 bits per element), or 16 when 32 would leave fewer
// than 1024 tiles to spread over the GPU
inline uint32_t auto_blocks_per_lane(int64_t nchunks) {
    return (nchunks + 32 * 32 - 1) / (32 * 32) >= 1024 ? 32u : 16u;
}

}  // namespace ta
}  // namespace ep
