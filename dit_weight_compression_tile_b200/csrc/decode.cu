// Fused tile decode for sm_100a: ep_decompress.
//
// The method's last stage ("EntroPack: Fast and Accurate Entropy-Coded Weight Compression at
// Arbitrary Bitrates", Abstract) is entropy coding in tiles that decode on their own, decoded on
// the GPU in the same pass that rebuilds the weights.  One kernel, one CTA per SM:
//   * ep_prepare (a small kernel, once per device copy of a stream) turns the frequency tables
//     into seven 2048-slot tables in a workspace.  A slot's 32-bit entry holds the token's
//     frequency (11 bits), the slot's offset inside the token (11 bits), an escape flag and, for
//     a direct token, the lattice coordinate v + 256 (9 bits).  Each decode CTA stages the 56 KB
//     with one bulk (TMA) copy;
//   * each warp decodes whole tiles.  A tile (32 initial states, 32 word counts, the lanes'
//     16-bit word streams, the raw extra bits) is brought into the warp's shared-memory buffer
//     by one bulk copy completing on an mbarrier, up to two tiles in flight per warp.  Lane l runs the
//     rANS coder of lane l over its own word stream, so a step is a table lookup, a
//     multiply-add and a predicated word read, with no warp-wide exchange;
//   * the coset c and the parity of y0..y6 that pick the contexts of coordinates 1..7 are bits
//     of the table entries, so a block's 8 tokens decode without a branch; the rare escape
//     tokens (a few per thousand) are resolved after the block from raw bits at the back of the
//     lane's word region;
//   * reconstruction stays in registers: the entry's value field becomes an exact float with
//     one logic op and one fused multiply-add, w = fp32(f_r * v) is one multiply, and the
//     container conversion rounds to nearest even; a warp stores 32 consecutive blocks with
//     one 16-byte (BF16 / FP16) or 8-byte (INT8 / FP8) store per lane.
// The path is a scan over compressed bytes, bound by HBM bandwidth and instruction issue; it
// uses no tensor cores because nothing in it is a dense contraction.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>
#include <mutex>

#include "../../include/eptile.h"
#include "device_util.cuh"
#include "format.h"

namespace ep {
namespace {

constexpr int kMaxWarps = 32;
constexpr uint32_t kSlotBytes = kProbScale * 4;                   // one context's slot table
constexpr size_t kLutBytes = size_t(kContexts) * kSlotBytes;      // 56 KB: the prepared tables
// A paired stream's tables: contexts 0 and 3..6 (slot tables, context 3 + 2c + p at position
// 1 + c + 2p), the pair tables of cosets 0 and 1 (4096 slots of 8 bytes), then 2 x 256 token
// fields for escaped pairs.
constexpr uint32_t kPairTabOff = 5 * kSlotBytes;
constexpr uint32_t kPairTabBytes = kPairScale * 8;
constexpr uint32_t kTokFieldOff = kPairTabOff + 2 * kPairTabBytes;
static_assert(kTokFieldOff + 2 * kPairTokFields * 4 == kPairedTableBytes, "paired table layout");
constexpr size_t kBarBytes = size_t(kMaxWarps) * 2 * 8 + 16;      // two mbarriers per warp + one for the tables
constexpr size_t kFixedBytes = kLutBytes + kBarBytes;
constexpr size_t kPairedFixedBytes = kPairedTableBytes + kBarBytes;
static_assert(kPairedFixedBytes % 16 == 0, "tile buffers must start 16-byte aligned");

// How a block's coordinates are coded, fixed per launch: one token each with value fields
// holding v (narrow) or y (wide), or coordinates 1..6 as three pair symbols (paired, narrow fields)
enum Coding { kNarrow = 0, kWide = 1, kPaired = 2 };
constexpr uint32_t kSlack = 160;      // bytes past a tile that a lane's bounded over-read may touch
                                      // (8 blocks of 8 tokens between checks, one word each, + 1)
constexpr size_t kSmemLimit = 232448; // shared memory one CTA may use on sm_100
static_assert(kFixedBytes % 16 == 0, "tile buffers must start 16-byte aligned");

// slot entry: bias [0,11) | value field [11,20) | escape [20] | frequency [21,32)
constexpr uint32_t kEscBit = 1u << 20;
constexpr uint32_t kFieldMask = 0x1ffu << 11;
// a direct token's entry becomes the float 2^34 + (v + 256) 2^22 with one OR; one FMA with
// 2^-22 and -(2^12 + 256) then gives v exactly
constexpr uint32_t kMagic = 0x50800000u;
constexpr float kInvScale = 1.0f / 4194304.0f;
constexpr float kBias = 4352.0f;

struct Params {
    const uint32_t *dir;     // tile directory, 16-byte units (T + 1 entries)
    const uint8_t *tiles;    // tile section
    const float *rowf;       // per-row factors f_r
    const uint32_t *tables;  // the stream's slot tables, prepared by ep_prepare (kLutBytes)
    void *out;               // container, row-major
    uint32_t *status;        // nullable
    uint64_t tile_units;     // size of the tile section in 16-byte units
    uint64_t cols;           // row length of the output in elements
    uint32_t nb;             // E8 blocks (rows * cb)
    uint32_t rows;
    uint32_t cb;             // blocks per row, ceil(cols / 8): a row is zero-padded to whole blocks
    uint32_t K;              // blocks per lane
    uint32_t T;              // tiles
    uint32_t tile_buf;       // bytes of each tile buffer (multiple of 16, includes kSlack)
    uint32_t nbuf;           // tile buffers per warp (1 or 2); 0: tiles are read from global memory
    uint32_t splits;         // 4 bits per context
    uint32_t pair_A[2];      // paired: token alphabet length of contexts 1 and 2
    uint32_t pair_rawb[2];   // paired: raw bits of one token of an escaped pair (<= 8)
};

// How a stream's blocks map onto rows, fixed per launch: kRowsAny (a lane's row is tested after
// every block), kRows32 (32 divides the blocks per row: a warp's step never straddles rows, so the
// loop runs row segment by row segment) and kRowsPadded (cols % 8 != 0: rows are zero-padded to
// whole E8 blocks and stores go element by element); kRowsGemm: the tiles are 128 x 64 operand
// tiles of a consumer GEMM (format.h lane_block), lane l taking row 32 (k mod 4) + l of its tile
// at column block k / 4, so each lane works on four rows whose factors it loads once per tile.
enum RowLayout { kRowsAny = 0, kRows32 = 1, kRowsPadded = 2, kRowsGemm = 3 };

__device__ __forceinline__ uint32_t split_of_bits(uint32_t splits, uint32_t c) { return (splits >> (4 * c)) & 15u; }
__device__ __forceinline__ uint32_t split_of(const Params &p, uint32_t c) { return split_of_bits(p.splits, c); }

__device__ __forceinline__ int32_t unzigzag(uint32_t u) { return int32_t(u >> 1) ^ -int32_t(u & 1u); }

// ------------------------------------------------------------------ containers
// put(i, v, w): coordinate i of the block, v the exact lattice value as a float and w = fp32(f_r v)
// the weight (one correctly rounded multiply), which the container rounds to nearest even.
template <int DT>
struct Packer;

// paired fp32 arithmetic of sm_100 (two independent IEEE operations, round to nearest each)
__device__ __forceinline__ uint64_t fma_x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul_x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t add_x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t pair(uint32_t lo, uint32_t hi) { return uint64_t(lo) | (uint64_t(hi) << 32); }

template <>
struct Packer<EP_BF16> {
    uint32_t o[4];
    float lo;
    __device__ __forceinline__ void put(int i, float, float w) {
        if (i & 1) {
            __nv_bfloat162 h = __floats2bfloat162_rn(lo, w);
            o[i >> 1] = *reinterpret_cast<uint32_t *>(&h);
        } else {
            lo = w;
        }
    }
    __device__ __forceinline__ void store(void *out, uint32_t b) {
        reinterpret_cast<uint4 *>(out)[b] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    // the 8 values as 16 bytes at a shared-memory address (an operand tile of the fused GEMM)
    __device__ __forceinline__ void store_shared(uint32_t a) {
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                     : "memory");
    }
    // the first n values at element e (the last block of a padded row: no vector store)
    __device__ __forceinline__ void store_n(void *out, uint64_t e, uint32_t n) {
        for (uint32_t i = 0; i < n; ++i)
            reinterpret_cast<uint16_t *>(out)[e + i] = uint16_t(o[i >> 1] >> (16 * (i & 1)));
    }
};

template <>
struct Packer<EP_FP16> {
    uint32_t o[4];
    float lo;
    __device__ __forceinline__ void put(int i, float, float w) {
        if (i & 1) {
            __half2 h = __floats2half2_rn(lo, w);
            o[i >> 1] = *reinterpret_cast<uint32_t *>(&h);
        } else {
            lo = w;
        }
    }
    __device__ __forceinline__ void store(void *out, uint32_t b) {
        reinterpret_cast<uint4 *>(out)[b] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __device__ __forceinline__ void store_n(void *out, uint64_t e, uint32_t n) {
        for (uint32_t i = 0; i < n; ++i)
            reinterpret_cast<uint16_t *>(out)[e + i] = uint16_t(o[i >> 1] >> (16 * (i & 1)));
    }
};

template <>
struct Packer<EP_FP32> {
    float o[8];
    __device__ __forceinline__ void put(int i, float, float w) { o[i] = w; }
    __device__ __forceinline__ void store(void *out, uint32_t b) {
        float4 *p = reinterpret_cast<float4 *>(out) + 2 * size_t(b);
        p[0] = make_float4(o[0], o[1], o[2], o[3]);
        p[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
    __device__ __forceinline__ void store_n(void *out, uint64_t e, uint32_t n) {
        for (uint32_t i = 0; i < n; ++i) reinterpret_cast<float *>(out)[e + i] = o[i];
    }
};

template <>
struct Packer<EP_INT8> {
    // clamp to [-127, 127] in fp32, then adding 1.5 * 2^23 rounds to the nearest integer (ties to
    // even) and leaves the code, two's complement, in the low byte of the sum's bits
    uint32_t b[8];
    __device__ __forceinline__ void put(int i, float, float w) {
        float r = __fadd_rn(fminf(fmaxf(w, -127.0f), 127.0f), 12582912.0f);
        b[i] = __float_as_uint(r);
    }
    // coordinates i and i + 1 at once: the two clamps, then one paired add
    __device__ __forceinline__ void put2(int i, uint64_t w2) {
        const float c0 = fminf(fmaxf(__uint_as_float(uint32_t(w2)), -127.0f), 127.0f);
        const float c1 = fminf(fmaxf(__uint_as_float(uint32_t(w2 >> 32)), -127.0f), 127.0f);
        const uint64_t r = add_x2(pair(__float_as_uint(c0), __float_as_uint(c1)),
                                  pair(__float_as_uint(12582912.0f), __float_as_uint(12582912.0f)));
        b[i] = uint32_t(r);
        b[i + 1] = uint32_t(r >> 32);
    }
    __device__ __forceinline__ uint2 packed() const {
        uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
        uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
        return make_uint2(lo, hi);
    }
    __device__ __forceinline__ void store(void *out, uint32_t blk) { reinterpret_cast<uint2 *>(out)[blk] = packed(); }
    // the 8 codes as 8 bytes at a shared-memory address (an operand slice of the fused GEMM)
    __device__ __forceinline__ void store_shared(uint32_t a) {
        const uint2 v = packed();
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(v.x), "r"(v.y) : "memory");
    }
    __device__ __forceinline__ void store_n(void *out, uint64_t e, uint32_t n) {
        for (uint32_t i = 0; i < n; ++i) reinterpret_cast<uint8_t *>(out)[e + i] = uint8_t(b[i]);
    }
};

template <>
struct Packer<EP_FP8_E4M3> {
    uint32_t o[2];
    float lo;
    __device__ __forceinline__ void put(int i, float, float w) {
        if (i & 1) {
            uint32_t pair = __nv_cvt_float2_to_fp8x2(make_float2(lo, w), __NV_SATFINITE, __NV_E4M3);
            if ((i & 3) == 1)
                o[i >> 2] = pair;
            else
                o[i >> 2] |= pair << 16;
        } else {
            lo = w;
        }
    }
    __device__ __forceinline__ void store(void *out, uint32_t b) {
        reinterpret_cast<uint2 *>(out)[b] = make_uint2(o[0], o[1]);
    }
    __device__ __forceinline__ void store_shared(uint32_t a) {
        asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(o[0]), "r"(o[1]) : "memory");
    }
    __device__ __forceinline__ void store_n(void *out, uint64_t e, uint32_t n) {
        for (uint32_t i = 0; i < n; ++i) reinterpret_cast<uint8_t *>(out)[e + i] = uint8_t(o[i >> 2] >> (8 * (i & 3)));
    }
};

// the lattice points themselves (v = 2z, int32), for consumers and bit-exact checks
template <>
struct Packer<EP_LATTICE_I32> {
    int32_t o[8];
    __device__ __forceinline__ void put(int i, float v, float) { o[i] = __float2int_rn(v); }
    __device__ __forceinline__ void store(void *out, uint32_t b) {
        int4 *p = reinterpret_cast<int4 *>(out) + 2 * size_t(b);
        p[0] = make_int4(o[0], o[1], o[2], o[3]);
        p[1] = make_int4(o[4], o[5], o[6], o[7]);
    }
    __device__ __forceinline__ void store_n(void *out, uint64_t e, uint32_t n) {
        for (uint32_t i = 0; i < n; ++i) reinterpret_cast<int32_t *>(out)[e + i] = o[i];
    }
};

// ------------------------------------------------------------------ a lane's words
// The tile's word area sits either in the warp's shared-memory buffer (SMEM) or, for a tile
// larger than any buffer, in global memory.  A lane keeps its state x, the next word w of its
// region (read ahead) and that word's address.  Raw extra bits are read from the back of the
// region.  Every address stays inside the buffer (shared memory: tile + slack) or the tile
// (global memory), whatever the stream holds.
template <bool SMEM>
struct Lane;

template <>
struct Lane<true> {
    uint32_t x, w;
    uint32_t wp;      // shared address of w
    uint32_t area;    // shared address of word 0 of the tile's word area
    uint32_t end;     // index one past the lane's region
    __device__ __forceinline__ void advance() {
        wp += 2;
        w = lds16(wp);
    }
    __device__ __forceinline__ bool past(uint32_t lim) const { return wp > lim; }
    __device__ __forceinline__ uint32_t word(int32_t i) const { return lds16(area + 2u * uint32_t(i)); }
    __device__ __forceinline__ uint32_t consumed(uint32_t start) const { return (wp - area) / 2u - start; }
};

template <>
struct Lane<false> {
    uint32_t x, w;
    const uint16_t *wp, *wlim;  // w's address; the last word this lane may touch
    const uint16_t *area;
    uint32_t end;
    __device__ __forceinline__ void advance() {
        wp = wp < wlim ? wp + 1 : wp;
        w = __ldg(wp);
    }
    // reads here are clamped to the tile one by one, so no block-level stop is needed
    __device__ __forceinline__ bool past(const uint16_t *) const { return false; }
    __device__ __forceinline__ uint32_t word(int32_t i) const { return __ldg(area + i); }
    __device__ __forceinline__ uint32_t consumed(uint32_t start) const { return uint32_t(wp - area) - start; }
};

// Below 2^16 the state takes the next word of the lane's region; the new state is stored.
template <bool SMEM>
__device__ __forceinline__ void renorm(Lane<SMEM> &L, uint32_t xn) {
    if constexpr (SMEM) {
        // predicated: x = x * 2^16 + w, then the next word of the region is read ahead
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.lt.u32 p, %0, 65536;\n\t@p mad.lo.u32 %0, %0, 65536, %2;\n\t"
            "@p add.u32 %1, %1, 2;\n\t@p ld.shared.u16 %2, [%1];\n\t}"
            : "+r"(xn), "+r"(L.wp), "+r"(L.w));
    } else if (xn < kStateLow) {
        xn = (xn << 16) | L.w;
        L.advance();
    }
    L.x = xn;
}

// One token of one lane: a lookup in the context's slot table and the rANS update
// x' = f (x >> 11) + (slot - cum); below 2^16 the state takes the next word of the region.
template <bool SMEM, bool ACT>
__device__ __forceinline__ uint32_t step(Lane<SMEM> &L, bool act, uint32_t lut) {
    if (ACT && !act) return 0u;
    // slot address lut + 4 (x mod 2^11) as two multiply-adds (lut + 4x - 2^13 (x >> 11), exact
    // modulo 2^32), which run on the FMA pipe beside the ALU work of the other lanes
    uint32_t xs = L.x >> kProbBits, a, t;
    asm("mad.lo.u32 %0, %1, 4, %2;" : "=r"(t) : "r"(L.x), "r"(lut));
    asm("mad.lo.u32 %0, %1, -8192, %2;" : "=r"(a) : "r"(xs), "r"(t));
    uint32_t e = lds32(a);
    uint32_t xn = (e >> 21) * xs + (e & (kProbScale - 1u));
    renorm(L, xn);
    return e;
}

// One pair symbol: a lookup in the coset's 4096-slot pair table of 8-byte entries (frequency
// [20,32) and slot offset [0,12), then the two coordinates' value fields at bits 11..20 and
// 21..30, or bit 31 for an escaped pair) and the update x' = f (x >> 12) + (slot - cum).
// Returns the entry's second word.
template <bool SMEM, bool ACT>
__device__ __forceinline__ uint32_t step2(Lane<SMEM> &L, bool act, uint32_t lutp) {
    if (ACT && !act) return 0u;
    // slot address lutp + 8 (x mod 2^12) = lutp + 8x - 2^15 (x >> 12), exact modulo 2^32
    uint32_t xs = L.x >> kPairBits, a, t, lo, hi;
    asm("mad.lo.u32 %0, %1, 8, %2;" : "=r"(t) : "r"(L.x), "r"(lutp));
    asm("mad.lo.u32 %0, %1, -32768, %2;" : "=r"(a) : "r"(xs), "r"(t));
    lds64(a, lo, hi);
    uint32_t xn = (lo >> 20) * xs + (lo & (kPairScale - 1u));
    renorm(L, xn);
    return hi;
}

// `nbits` raw bits at raw-bit position rb of the lane (the region's last word holds bits
// 0..15), least significant first; nbits <= 19 and rb is clamped by the caller so that the three
// words read lie inside the tile (shared memory: inside the buffer)
template <bool SMEM>
__device__ __forceinline__ uint32_t raw_bits(const Lane<SMEM> &L, uint32_t rb, uint32_t nbits) {
    int32_t j = int32_t(L.end) - 1 - int32_t(rb >> 4);
    uint32_t lo = __byte_perm(L.word(j), L.word(j - 1), 0x5410);  // bits rb & ~15 .. + 31
    uint32_t hi = L.word(j - 2);
    return __funnelshift_r(lo, hi, rb & 15u) & ((1u << nbits) - 1u);
}

// Escape tokens of a block (the warp has at least one).  Token layout (split m, `low` kept
// bits, 2 bits below the leading one): d = token - 2^m = ((n - m) << 2 | top) << low | lo; the
// value is s = (4 | top) << (n - 2) | extra << low | lo with n - 2 - low raw extra bits.  F[i]
// holds the entry's value field (d, or 2d + c for coordinates 1..6) and its escape flag.
template <bool SMEM, bool WIDE>
__device__ __forceinline__ void resolve_escapes(const Params &p, uint32_t (&F)[8], uint32_t c, uint32_t par,
                                                Lane<SMEM> &L, uint32_t &rb) {
    uint32_t lm = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) lm |= ((F[i] >> 20) & 1u) << i;
    uint32_t M = __reduce_or_sync(0xffffffffu, lm);
    // a damaged region cannot move the raw reads below the tile's head
    rb = min(rb, 16u * (L.end + 88u));
    const uint32_t m0 = split_of(p, 0), m16 = split_of(p, 1u + c), m7 = split_of(p, 3u + 2u * c + par);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (M & (1u << i)) {
            if (lm & (1u << i)) {
                const uint32_t low = i == 0 ? 2u : (i < 7 ? 1u : 0u);
                uint32_t m = i == 0 ? m0 : (i < 7 ? m16 : m7);
                uint32_t fld = (F[i] >> 11) & 0x1ffu;
                uint32_t d = (!WIDE && i >= 1 && i <= 6) ? fld >> 1 : fld;
                uint32_t q = d >> low;
                uint32_t n = min(m + (q >> 2), kValueBits - 1u);
                uint32_t nbits = n - 2u - low;
                uint32_t extra = raw_bits(L, rb, nbits);
                rb += nbits;
                uint32_t s = ((4u | (q & 3u)) << (n - 2u)) | (extra << low) | (d & ((1u << low) - 1u));
                int32_t v;
                if (i == 0)
                    v = 4 * unzigzag(s >> 2) + int32_t(s & 3u);
                else if (i < 7)
                    v = 2 * (2 * unzigzag(s >> 1) + int32_t(s & 1u)) + int32_t(c);
                else
                    v = 2 * (2 * unzigzag(s) + int32_t(par)) + int32_t(c);
                // the word the reconstruction expects: v (coordinate 0, narrow tables) or
                // y = (v - c) / 2 (coordinates 1..7 of wide tables), plus 4352, times 2^22
                const int32_t u = (WIDE && i > 0) ? (v - int32_t(c)) >> 1 : v;
                F[i] = __float_as_uint(__int2float_rn(u + 4352) * 4194304.0f);
            }
        }
    }
}

// Escaped pairs of a block (the warp has at least one): their two tokens are the first raw bits of
// the block, pair by pair, each in p.pair_rawb[c] bits; the value fields come from the coset's
// token-field table.  A token beyond the alphabet is reported (the index stays inside the table).
template <bool SMEM>
__device__ __forceinline__ uint32_t resolve_pair(const Params &p, uint32_t h, uint32_t c, uint32_t tf,
                                                 const Lane<SMEM> &L, uint32_t &rb, uint32_t &err) {
    if (!(h >> 31)) return h;
    // a damaged region cannot move the raw reads below the tile's head
    rb = min(rb, 16u * (L.end + 88u));
    const uint32_t nb = p.pair_rawb[c];
    const uint32_t bits = raw_bits(L, rb, 2u * nb);
    rb += 2u * nb;
    const uint32_t ta = bits & ((1u << nb) - 1u), tb = bits >> nb;
    if (ta >= p.pair_A[c] || tb >= p.pair_A[c]) err |= EP_DEC_BAD_TOKEN;
    return lds32(tf + 4u * (ta & (kPairTokFields - 1u))) | (lds32(tf + 4u * (tb & (kPairTokFields - 1u))) << 10);
}

// ------------------------------------------------------------------ the blocks of one tile
// Lane l decodes blocks t*32K + 32k + l, k = 0..K-1.  ACT: the last tile, where lanes run out
// of blocks.  ROWS: the launch's RowLayout.  Returns EP_DEC_* bits.
// Sink (GEMM-ordered BF16 / INT8 / FP8 tiles only; NoSink otherwise): the blocks go to shared-memory
// operand slices of the fused GEMM instead of global memory.  sink.begin(k) runs before step k (it may
// wait for a buffer; false gives up), sink.put(k, lane, pk) stores the step's 8 weights and
// sink.end(k, lane) runs after the store.
struct NoSink {};

template <int DT, bool SMEM, bool ACT, int ROWS, int MODE, typename Lim, typename Sink = NoSink>
__device__ __forceinline__ uint32_t decode_blocks(const Params &p, Lane<SMEM> &L, uint32_t &rb, uint32_t lut,
                                                  Lim wlim, uint32_t t, uint32_t lane, Sink *sink = nullptr) {
    constexpr bool TO_SMEM = !std::is_same<Sink, NoSink>::value;
    constexpr bool WIDE = MODE == kWide;
    constexpr bool R32 = ROWS == kRows32, RAG = ROWS == kRowsPadded, GEMM = ROWS == kRowsGemm;
    uint32_t b = t * 32u * p.K + lane;
    uint32_t row = b / p.cb, col = b - row * p.cb;
    // the factor of the current row and of the next one (read a row ahead)
    float fr = 0.0f, frn = 0.0f;
    // GEMM tiles: the lane's four rows r0 + 32 j and their factors; block k sits at
    // (r0 + 32 (k mod 4)) cb + c0 + k / 4
    float fg0 = 0.0f, fg1 = 0.0f, fg2 = 0.0f, fg3 = 0.0f;
    uint32_t gbase = 0;
    if constexpr (GEMM) {
        const uint32_t kt = p.cb >> 3, r0 = 128u * (t / kt) + lane;
        gbase = r0 * p.cb + 8u * (t % kt);
        fg0 = __ldg(p.rowf + r0);
        fg1 = __ldg(p.rowf + r0 + 32);
        fg2 = __ldg(p.rowf + r0 + 64);
        fg3 = __ldg(p.rowf + r0 + 96);
    } else {
        fr = row < p.rows ? __ldg(p.rowf + row) : 0.0f;
        frn = row + 1 < p.rows ? __ldg(p.rowf + row + 1) : 0.0f;
    }
    uint32_t err = 0;
    uint32_t k = 0;
    for (;;) {
        // R32 (32 | blocks per row): the warp's 32 blocks of a step lie in one row, so all lanes
        // change rows after the same number of steps and the step loop needs no row test
        uint32_t kseg = p.K;
        if constexpr (R32) {
            uint32_t left = (p.cb - (col - lane)) >> 5;
            kseg = k + left < p.K ? k + left : p.K;
        }
        for (; k < kseg; ++k, b += 32u) {
            if constexpr (GEMM) {
                b = gbase + (k & 3u) * 32u * p.cb + (k >> 2);
                fr = (k & 2u) ? ((k & 1u) ? fg3 : fg2) : ((k & 1u) ? fg1 : fg0);
            }
            bool act = !ACT || b < p.nb;
            if (ACT && !__any_sync(0xffffffffu, act)) goto done;
            if constexpr (TO_SMEM) {
                if (!sink->begin(k)) {
                    err |= EP_DEC_TIMEOUT;
                    goto done;
                }
            }
            // a damaged stream may drive a lane's reads ahead (at most one word per token); stop
            // before they leave the buffer's slack
            if ((k & 7u) == 0 && __any_sync(0xffffffffu, L.past(wlim))) {
                err |= EP_DEC_WORD_OVERRUN;
                goto done;
            }
            // F keeps the value field and the escape flag of each coordinate (the flag only matters
            // for escapes, whose F is rebuilt), so the entries themselves die early
            uint32_t F[8], Y;
            if constexpr (MODE == kPaired) {
                // token 0, the pairs (1,2), (3,4), (5,6) from the coset's pair table, token 7.
                // The pair entries carry the same value fields as token entries, so bits 11 and
                // 12 of the XOR of all seven fields are again c and the parity p of y0..y6
                const uint32_t e0 = step<SMEM, ACT>(L, act, lut);
                const uint32_t lutp = lut + kPairTabOff + ((e0 & 0x800u) << 4);  // pair table of c
                uint32_t h0 = step2<SMEM, ACT>(L, act, lutp);
                uint32_t h1 = step2<SMEM, ACT>(L, act, lutp);
                uint32_t h2 = step2<SMEM, ACT>(L, act, lutp);
                if (__any_sync(0xffffffffu, (h0 | h1 | h2) >> 31)) {
                    const uint32_t c = (e0 >> 11) & 1u, tf = lut + kTokFieldOff + 4u * kPairTokFields * c;
                    h0 = resolve_pair(p, h0, c, tf, L, rb, err);
                    h1 = resolve_pair(p, h1, c, tf, L, rb, err);
                    h2 = resolve_pair(p, h2, c, tf, L, rb, err);
                }
                const uint32_t H = h0 ^ h1 ^ h2;
                Y = (e0 ^ H ^ (H >> 10)) & 0x1800u;
                // context 3 + 2c + p sits at table position 1 + c + 2p
                const uint32_t e7 = step<SMEM, ACT>(L, act, lut + kSlotBytes + (Y << 2));
                F[0] = (e0 & (kFieldMask | kEscBit)) | kMagic;
                F[1] = (h0 & (kFieldMask | kEscBit)) | kMagic;
                F[2] = ((h0 >> 10) & (kFieldMask | kEscBit)) | kMagic;
                F[3] = (h1 & (kFieldMask | kEscBit)) | kMagic;
                F[4] = ((h1 >> 10) & (kFieldMask | kEscBit)) | kMagic;
                F[5] = (h2 & (kFieldMask | kEscBit)) | kMagic;
                F[6] = ((h2 >> 10) & (kFieldMask | kEscBit)) | kMagic;
                F[7] = (e7 & (kFieldMask | kEscBit)) | kMagic;
            } else {
                uint32_t e[8];
                // coordinate 0 (context 0); bit 11 of every entry of contexts 0..2 is the coset c
                e[0] = step<SMEM, ACT>(L, act, lut);
                uint32_t lutc = lut + kSlotBytes + ((e[0] & 0x800u) << 2);  // context 1 + c
#pragma unroll
                for (int i = 1; i < 7; ++i) e[i] = step<SMEM, ACT>(L, act, lutc);
                // narrow tables: bits 11 and 12 of the XOR of entries 0..6 are c (seven copies) and
                // the parity p of y0..y6.  Wide tables: bit 11 of entries 1..6 is the parity of y_i,
                // so c is bit 11 of entry 0 and p is bit 12 of entry 0 xor bit 11 of the others' XOR.
                // Context 3 + 2c + p sits at table position 3 + c + 2p
                if constexpr (WIDE) {
                    const uint32_t X1 = e[1] ^ e[2] ^ e[3] ^ e[4] ^ e[5] ^ e[6];
                    Y = (e[0] & 0x800u) | ((e[0] ^ (X1 << 1)) & 0x1000u);
                } else {
                    Y = (e[0] ^ e[1] ^ e[2] ^ e[3] ^ e[4] ^ e[5] ^ e[6]) & 0x1800u;
                }
                uint32_t lut7 = lut + 3u * kSlotBytes + (Y << 2);
                e[7] = step<SMEM, ACT>(L, act, lut7);
#pragma unroll
                for (int i = 0; i < 8; ++i) F[i] = (e[i] & (kFieldMask | kEscBit)) | kMagic;
            }
            const uint32_t cbit = (Y >> 11) & 1u, pbit = (Y >> 12) & 1u;
            uint32_t O = F[0] | F[1] | F[2] | F[3] | F[4] | F[5] | F[6] | F[7];
            if (__any_sync(0xffffffffu, O & kEscBit))
                resolve_escapes<SMEM, WIDE>(p, F, cbit, pbit, L, rb);
            // v = F 2^-22 - (2^12 + 256) exactly, w = fp32(f_r v): two coordinates per instruction
            // narrow: v = F 2^-22 - 4352 for every coordinate; wide: coordinates 1..7 hold y, and
            // v = 2 y + c = F 2^-21 - 8704 + c (exact: integers below 2^24)
            const uint64_t scale2 = WIDE ? pair(__float_as_uint(2.0f * kInvScale), __float_as_uint(2.0f * kInvScale))
                                         : pair(__float_as_uint(kInvScale), __float_as_uint(kInvScale));
            const float bw = cbit ? -2.0f * kBias + 1.0f : -2.0f * kBias;
            const uint64_t bias2 = WIDE ? pair(__float_as_uint(bw), __float_as_uint(bw))
                                        : pair(__float_as_uint(-kBias), __float_as_uint(-kBias));
            const uint64_t scale01 = WIDE ? pair(__float_as_uint(kInvScale), __float_as_uint(2.0f * kInvScale)) : scale2;
            const uint64_t bias01 = WIDE ? pair(__float_as_uint(-kBias), __float_as_uint(bw)) : bias2;
            const uint64_t fr2 = pair(__float_as_uint(fr), __float_as_uint(fr));
            Packer<DT> pk;
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                uint64_t v2 = fma_x2(pair(F[i], F[i + 1]), i == 0 ? scale01 : scale2, i == 0 ? bias01 : bias2);
                uint64_t w2 = mul_x2(v2, fr2);
                if constexpr (DT == EP_INT8) {
                    pk.put2(i, w2);
                } else {
                    pk.put(i, __uint_as_float(uint32_t(v2)), __uint_as_float(uint32_t(w2)));
                    pk.put(i + 1, __uint_as_float(uint32_t(v2 >> 32)), __uint_as_float(uint32_t(w2 >> 32)));
                }
            }
            if constexpr (RAG) {
                // a padded row's last block keeps its first cols % 8 values
                const uint64_t c0 = 8ull * col;
                if (act) pk.store_n(p.out, uint64_t(row) * p.cols + c0, uint32_t(min(p.cols - c0, uint64_t(8))));
            } else if constexpr (TO_SMEM) {
                static_assert((DT == EP_BF16 || DT == EP_INT8 || DT == EP_FP8_E4M3) && ROWS == kRowsGemm,
                              "operand slices come from GEMM-ordered BF16 / INT8 / FP8 tiles");
                sink->put(k, lane, pk);
                sink->end(k, lane);
            } else if (act) {
                pk.store(p.out, b);
            }
            if constexpr (!R32 && !GEMM) {
                col += 32u;
                if (col >= p.cb) {  // next row
                    col -= p.cb;
                    ++row;
                    fr = frn;
                    while (col >= p.cb) {
                        col -= p.cb;
                        ++row;
                        fr = row < p.rows ? __ldg(p.rowf + row) : 0.0f;
                    }
                    frn = row + 1 < p.rows ? __ldg(p.rowf + row + 1) : 0.0f;
                }
            }
        }
        if (!R32 || k >= p.K) break;
        // the segment ended at the end of the row: the next step starts the next row at column lane
        col = lane;
        ++row;
        fr = frn;
        frn = row + 1 < p.rows ? __ldg(p.rowf + row + 1) : 0.0f;
    }
done:
    return err;
}

// Decodes tile t with one warp.  `head` points at the tile (states, region lengths, word area):
// a shared address (SMEM) or a global pointer.  Returns the EP_DEC_* bits of this lane.
template <int DT, int ROWS, int MODE, bool SMEM, typename Ptr, typename Sink = NoSink>
__device__ __forceinline__ uint32_t decode_tile(const Params &p, uint32_t lut, Ptr head, uint32_t tile_bytes,
                                                uint32_t t, uint32_t lane, Sink *sink = nullptr) {
    constexpr bool TO_SMEM = !std::is_same<Sink, NoSink>::value;
    Lane<SMEM> L;
    uint32_t len;
    if constexpr (SMEM) {
        L.x = lds32(head + 4u * lane);
        len = lds16(head + 128u + 2u * lane);
    } else {
        L.x = __ldg(reinterpret_cast<const uint32_t *>(head) + lane);
        len = __ldg(reinterpret_cast<const uint16_t *>(head + 128) + lane);
    }
    // each lane's region starts after the lower lanes' regions
    uint32_t incl = len;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= uint32_t(d)) incl += y;
    }
    uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t capacity = (tile_bytes - uint32_t(kTileHead)) / 2u;
    if (total > capacity) return EP_DEC_WORD_OVERRUN;  // warp-uniform: the regions overrun the tile
    uint32_t start = incl - len;
    L.end = incl;
    uint32_t rb = 0, err;
    if constexpr (SMEM) {
        L.area = head + uint32_t(kTileHead);
        L.wp = L.area + 2u * start;
        L.w = lds16(L.wp);
        uint32_t wlim = L.area + 2u * capacity;
        if (TO_SMEM || uint64_t(t + 1) * 32u * p.K <= p.nb)
            err = decode_blocks<DT, SMEM, false, ROWS, MODE, uint32_t, Sink>(p, L, rb, lut, wlim, t, lane, sink);
        else
            err = decode_blocks<DT, SMEM, true, ROWS, MODE>(p, L, rb, lut, wlim, t, lane);
    } else {
        L.area = reinterpret_cast<const uint16_t *>(head + kTileHead);
        L.wlim = L.area + (capacity ? capacity - 1u : 0u);
        L.wp = L.area + start < L.wlim ? L.area + start : L.wlim;
        L.w = __ldg(L.wp);
        if (uint64_t(t + 1) * 32u * p.K <= p.nb)
            err = decode_blocks<DT, SMEM, false, ROWS, MODE>(p, L, rb, lut, L.wlim, t, lane);
        else
            err = decode_blocks<DT, SMEM, true, ROWS, MODE>(p, L, rb, lut, L.wlim, t, lane);
    }
    if (L.x != kStateLow) err |= EP_DEC_BAD_END;
    // the front (rANS words) and the back (raw bits) cover the region exactly
    uint32_t used = L.consumed(start) + (rb + 15u) / 16u;
    if (used != len) err |= used > len ? EP_DEC_WORD_OVERRUN : EP_DEC_WORD_COUNT;
    if (capacity - total >= 8u) err |= EP_DEC_WORD_COUNT;
    return err;
}

// ------------------------------------------------------------------ slot tables
// Entry of token t of context c with frequency f: frequency, escape flag and value field (the
// offset of the slot inside the token is added per slot).  A direct token stores v + 256 of
// the coordinate it stands for; an escape token stores its index past 2^m (for coordinates
// 1..6 as 2 d + c, so that bits 0 and 1 of the field are the coset and the parity of y in
// every entry of contexts 0..2).
__device__ __forceinline__ uint32_t token_head(uint32_t c, uint32_t t, uint32_t f, uint32_t m, bool wide) {
    uint32_t field;
    if (t < (1u << m)) {
        int32_t v;  // narrow tables: the coordinate v; wide tables: y = (v - c) / 2 for coordinates 1..7
        if (c == 0)
            v = 4 * unzigzag(t >> 2) + int32_t(t & 3u);
        else if (c < 3)
            v = wide ? 2 * unzigzag(t >> 1) + int32_t(t & 1u)
                     : 2 * (2 * unzigzag(t >> 1) + int32_t(t & 1u)) + int32_t(c - 1);
        else
            v = wide ? 2 * unzigzag(t) + int32_t((c - 3) & 1u)
                     : 2 * (2 * unzigzag(t) + int32_t((c - 3) & 1u)) + int32_t((c - 3) >> 1);
        field = (uint32_t(v + 256) & 0x1ffu) << 11;
    } else {
        uint32_t d = t - (1u << m);
        uint32_t fv = (!wide && (c == 1 || c == 2)) ? 2u * d + (c - 1) : d;
        field = kEscBit | ((fv & 0x1ffu) << 11);
    }
    return (min(f, kProbScale - 1u) << 21) | field;
}

// ------------------------------------------------------------------ ep_prepare: the slot tables
// One CTA per (context, 256 slots): the context's frequencies and their prefix sums in shared
// memory, then each thread finds the symbol of its slot by binary search.  Runs once per stream;
// the decode kernel copies the result (56 KB; a paired stream's 106 KB) into every CTA's
// shared memory.  Grid: 7 contexts x 8 CTAs; paired streams: contexts 0, 3..6 x 8 CTAs, then
// the pair tables of contexts 1, 2 x 16 CTAs (4096 slots each).
struct PrepParams {
    const uint16_t *freq;    // frequency tables, contexts in order
    uint32_t *tables;        // the decoder's tables (kLutBytes, or kPairedTableBytes when paired)
    uint32_t *status;        // nullable
    uint32_t splits;
    uint32_t wide;           // value fields hold y for coordinates 1..7
    uint32_t paired;
    uint32_t ntok[kContexts];
    uint32_t tab_off[kContexts + 1];
};

constexpr uint32_t kPrepThreads = 256;
constexpr uint32_t kPrepSingleCtas = kProbScale / kPrepThreads;  // 8 per token table
constexpr uint32_t kPrepPairCtas = kPairScale / kPrepThreads;    // 16 per pair table

// value field and escape flag (bits 11..20) of token t of context c
__device__ __forceinline__ uint32_t token_field(uint32_t c, uint32_t t, uint32_t m, bool wide) {
    return token_head(c, t, 0u, m, wide) & (kFieldMask | kEscBit);
}

__global__ void __launch_bounds__(kPrepThreads) prepare_kernel(const __grid_constant__ PrepParams p) {
    __shared__ uint32_t cum[kPairMaxTable + 1];
    __shared__ uint32_t part[kPrepThreads / 32];
    uint32_t c, slot0;
    bool pair = false;
    if (!p.paired) {
        c = blockIdx.x / kPrepSingleCtas;
        slot0 = (blockIdx.x % kPrepSingleCtas) * kPrepThreads;
    } else if (blockIdx.x < 5 * kPrepSingleCtas) {
        const uint32_t i = blockIdx.x / kPrepSingleCtas;
        c = i == 0 ? 0u : i + 2u;
        slot0 = (blockIdx.x % kPrepSingleCtas) * kPrepThreads;
    } else {
        const uint32_t j = blockIdx.x - 5 * kPrepSingleCtas;
        c = 1u + j / kPrepPairCtas;
        slot0 = (j % kPrepPairCtas) * kPrepThreads;
        pair = true;
    }
    const uint32_t M = pair ? kPairScale : kProbScale;
    const uint32_t slot = slot0 + threadIdx.x;
    const uint32_t n = min(p.tab_off[c + 1] - p.tab_off[c], pair ? kPairMaxTable : kMaxAlphabet);
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    // exclusive prefix sums of the (clamped) frequencies, 256 at a time
    uint32_t run = 0;
    bool bad = false;
    for (uint32_t base = 0; base < n; base += kPrepThreads) {
        uint32_t t = base + threadIdx.x;
        uint32_t f = t < n ? uint32_t(p.freq[p.tab_off[c] + t]) : 0u;
        bad |= f >= M;
        f = min(f, M);
        uint32_t incl = f;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= uint32_t(d)) incl += y;
        }
        if (lane == 31) part[warp] = incl;
        __syncthreads();
        uint32_t before = 0, all = 0;
        for (uint32_t w = 0; w < kPrepThreads / 32; ++w) {
            before += w < warp ? part[w] : 0u;
            all += part[w];
        }
        if (t < n) cum[t] = min(run + before + incl - f, 0xffffu);
        run = min(run + all, 0xffffu);
        __syncthreads();
    }
    if (threadIdx.x == 0) cum[n] = run;
    __syncthreads();
    if (p.status && slot0 == 0 && threadIdx.x == 0 && n && run != M) atomicOr(p.status, EP_DEC_BAD_TOKEN);
    if (p.status && __syncthreads_or(bad) && threadIdx.x == 0) atomicOr(p.status, EP_DEC_BAD_TOKEN);
    // the last symbol s with cum[s] <= slot (symbols with f = 0 are skipped)
    uint32_t sym = 0, f = 0;
    if (n) {
        uint32_t lo = 0, hi = n;  // cum[lo] <= slot < cum[hi] (cum[n] may be short if damaged)
        while (hi - lo > 1) {
            uint32_t mid = (lo + hi) >> 1;
            if (cum[mid] <= slot)
                lo = mid;
            else
                hi = mid;
        }
        sym = lo;
        f = cum[lo + 1] - cum[lo];
    }
    const uint32_t m = split_of_bits(p.splits, c);
    if (!pair) {
        uint32_t e = n ? token_head(c, sym, f, m, p.wide != 0) | ((slot - cum[sym]) & (kProbScale - 1u)) : 0u;
        // context 3 + 2c + p is stored at position 3 + c + 2p (1 + c + 2p in a paired stream's
        // tables); the decoder forms that offset from the XOR of a block's first seven fields
        const uint32_t first = p.paired ? 1u : 3u;
        uint32_t pos = c < 3 ? c : first + ((c - 3u) >> 1) + 2u * ((c - 3u) & 1u);
        p.tables[pos * kProbScale + slot] = e;
    } else {
        // pair entry: frequency and slot offset, then the fields of tokens (t_a, t_b) = (s / B, s % B)
        // or bit 31 for the escape symbol s = B * B (B = min(A, 40))
        const uint32_t A = p.ntok[c], B = min(A, kPairBaseMax);
        uint32_t lo = 0, hi = 0;
        if (n) {
            lo = (min(f, kPairScale - 1u) << 20) | ((slot - cum[sym]) & (kPairScale - 1u));
            hi = sym >= B * B ? (1u << 31)
                              : token_field(c, sym / B, m, false) | (token_field(c, sym % B, m, false) << 10);
        }
        uint32_t *dst = p.tables + (kPairTabOff + (c - 1u) * kPairTabBytes) / 4u + 2u * slot;
        dst[0] = lo;
        dst[1] = hi;
        if (slot < kPairTokFields)
            p.tables[kTokFieldOff / 4u + (c - 1u) * kPairTokFields + slot] = slot < A ? token_field(c, slot, m, false) : 0u;
    }
}

// ------------------------------------------------------------------ decode kernel
// Shared memory: the slot tables, mbarriers, then nbuf tile buffers per warp.
template <int DT, int ROWS, int MODE>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) decode_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr uint32_t kTables = uint32_t(MODE == kPaired ? kPairedTableBytes : kLutBytes);
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const uint32_t lut = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const uint32_t bars = lut + kTables;
    const uint32_t tbar = bars + uint32_t(kMaxWarps) * 16u;  // the tables' mbarrier
    const uint32_t nbuf = p.nbuf;
    const uint32_t bufs = bars + uint32_t(kBarBytes) + warp * (nbuf ? nbuf : 1u) * p.tile_buf;
    const uint32_t t_begin = uint32_t(uint64_t(blockIdx.x) * p.T / gridDim.x);
    const uint32_t t_end = uint32_t(uint64_t(blockIdx.x + 1) * p.T / gridDim.x);

    if (threadIdx.x == 0) {
        for (uint32_t w = 0; w < nwarps; ++w) {
            mbar_init(bars + 16u * w, 1);
            mbar_init(bars + 16u * w + 8u, 1);
        }
        mbar_init(tbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async();
    }
    // launched with programmatic stream serialisation: the CTA may start while the previous kernel
    // of the stream drains; nothing global is touched before that kernel's writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        mbar_expect(tbar, kTables);
        bulk_g2s(lut, p.tables, kTables, tbar);
    }
    __syncthreads();

    // a tile's copy into buffer j of this warp; every lane computes whether it was issued
    auto tile_ok = [&](uint32_t t, uint32_t &beg, uint32_t &bytes) -> bool {
        beg = __ldg(p.dir + t);
        uint32_t end = __ldg(p.dir + t + 1);
        bytes = (end - beg) * 16u;
        return end >= beg + uint32_t(kTileHead / 16) && uint64_t(end) <= p.tile_units;
    };
    auto issue = [&](uint32_t t, uint32_t j) -> bool {
        uint32_t beg, bytes;
        bool ok = tile_ok(t, beg, bytes) && nbuf && bytes + kSlack <= p.tile_buf;
        if (ok && lane == 0) {
            uint32_t bar = bars + 16u * warp + 8u * j;
            fence_proxy_async();
            mbar_expect(bar, bytes);
            bulk_g2s(bufs + j * p.tile_buf, p.tiles + size_t(beg) * 16, bytes, bar);
        }
        return ok;
    };
    // per buffer: a copy in flight (bit 0 / 1) and the mbarrier phase to wait for (bit 0 / 1)
    uint32_t pend = 0, phase = 0;
    for (uint32_t j = 0; j < nbuf; ++j) {
        uint32_t t = t_begin + warp + j * nwarps;
        if (t < t_end && issue(t, j)) pend |= 1u << j;
    }
    bool tables_ok = mbar_wait(tbar, 0);
    if (!tables_ok && lane == 0 && p.status) atomicOr(p.status, EP_DEC_TIMEOUT);

    // ---- tiles of this CTA: a contiguous range, warps round robin, nbuf copies in flight
    uint32_t j = 0;
    for (uint32_t t = t_begin + warp; t < t_end; t += nwarps, ++j) {
        uint32_t b = nbuf ? j % nbuf : 0u;
        uint32_t beg, bytes, err = 0;
        bool valid = tile_ok(t, beg, bytes);
        if (!valid) {
            err = EP_DEC_BAD_TILE;
        } else if (pend & (1u << b)) {
            bool done = mbar_wait(bars + 16u * warp + 8u * b, (phase >> b) & 1u);
            phase ^= 1u << b;
            pend &= ~(1u << b);
            if (!done) {  // a lost copy: report, let the other buffer's copy land, stop
                if (lane == 0 && p.status) atomicOr(p.status, EP_DEC_TIMEOUT);
                uint32_t o = b ^ 1u;
                if (nbuf > 1 && (pend & (1u << o))) mbar_wait(bars + 16u * warp + 8u * o, (phase >> o) & 1u);
                return;
            }
            if (tables_ok) err = decode_tile<DT, ROWS, MODE, true>(p, lut, bufs + b * p.tile_buf, bytes, t, lane);
        } else if (tables_ok) {
            err = decode_tile<DT, ROWS, MODE, false>(p, lut, p.tiles + size_t(beg) * 16, bytes, t, lane);
        }
        if (err && p.status) atomicOr(p.status, err);
        __syncwarp();
        uint32_t tn = t + nbuf * nwarps;
        if (nbuf && tn < t_end && issue(tn, b)) pend |= 1u << b;
    }
}

// ------------------------------------------------------------------ the decode fused into a GEMM
// Y^T = W X^T for a weight W (N x K) held as a GEMM-ordered stream (EP_LAYOUT_GEMM): each stream tile
// is one 128 x 64 tile of W.  One CTA per (band of 128 output features, range of K tiles); warps
// 0 .. S-1 decode, one tile at a time each: a bulk copy of the stream tile into the warp's buffer,
// the matching slice of X (tokens padded to a multiple of 16) into the warp's X buffer, then the
// tile's 32 steps.  Every 8 steps complete a 128 x 16 K-slice of the tile, which goes to one of the
// warp's two 4 KB slice buffers (a ring) and is announced on that buffer's `full` barrier.  Warp S
// issues the tensor-core work: for each round of tiles, slice by slice, warp by warp (a fixed
// order, so the fp32 sums are the same on every call), one tcgen05.mma (M = 128 features,
// N = tokens, K = 16, A = the W slice, B = the X slice, both K-major) accumulating in tensor
// memory, committed to the slice buffer's `empty` barrier.  After the last MMA, warps 0..3 read
// the 128 x N fp32 accumulator out of tensor memory into the CTA's slice of the partial sums; the
// band's last CTA to finish adds the splits' partial sums in split order (the same sums on every
// call), adds the bias, rounds once to BF16 and writes Y.
constexpr uint32_t kLinMaxWarps = 15;       // decoding warps per CTA
constexpr uint32_t kLinSlice = 128u * 16u * 2u;  // one 128 x 16 BF16 K-slice of a W tile
constexpr uint32_t kLinBarBytes = 40;       // per decoding warp: full[2], empty[2], copy

struct LinParams {
    Params dp;                 // the stream (tiles, tables, row factors, status)
    const uint16_t *x;         // activations, BF16, M x cols row-major
    float *part;               // fp32 partial sums, splits x M x N
    uint32_t *count;           // per band: CTAs done (zero between calls)
    const uint16_t *bias;      // nullable, BF16, N
    uint16_t *y;               // BF16, M x N
    uint32_t splits;
    const uint8_t *xq;         // code containers: the activations' 8-bit codes, M x cols
    const float *xscale;       // code containers: the activations' per-token scales
    const float *wscale;       // code containers: the weight's per-row scales (from the stream)
    uint32_t M, N;             // tokens, output features (rows of W)
    uint32_t npad;             // tokens padded to a multiple of 16 (the MMA's N)
    uint32_t idesc;            // the MMA's instruction descriptor
    uint32_t tmem_cols;        // tensor-memory columns of the accumulator (a power of 2, >= 32)
    uint32_t KT;               // K tiles per band (cols / 64)
    uint32_t kt_per_split;
    uint32_t S;                // decoding warps
    uint32_t tile_buf;         // bytes of a stream-tile buffer
    uint32_t off_bars, off_tile, off_w, off_x;  // shared-memory layout (offsets from the dynamic base)
};

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// UMMA shared-memory descriptor of a K-major operand without swizzle at shared address a: 8 x 16-byte
// core matrices, `lbo` bytes apart along K and `sbo` bytes apart along M / N (both in 16-byte
// units), descriptor version 1, layout type 0
__device__ __forceinline__ uint64_t umma_desc_plain(uint32_t a, uint32_t lbo, uint32_t sbo) {
    return uint64_t((a >> 4) & 0x3fffu) | (uint64_t((lbo >> 4) & 0x3fffu) << 16) |
           (uint64_t((sbo >> 4) & 0x3fffu) << 32) | (uint64_t(1) << 46);
}

// where a decoding warp's steps go.  A K-slice is 128 rows x 32 bytes of the tile (16 BF16 weights or
// 32 8-bit codes: the K extent of one MMA), stored as no-swizzle K-major core matrices: row r's
// 16-byte chunk c at (r / 8) 256 + 128 c + 16 (r mod 8).  Step k writes 8 weights of row
// 32 (k mod 4) + lane at column block k / 4, so BF16 tiles complete a slice every 8 steps (4 slices
// per tile), 8-bit tiles every 16 (2 slices); slice j of the warp's round-th tile is its use
// U round + j (U slices per tile) and lives in ring buffer j mod 2.
template <int DT>
struct SliceSink {
    static constexpr uint32_t kSteps = DT == EP_BF16 ? 8u : 16u;  // steps per slice
    static constexpr uint32_t kUses = 32u / kSteps;                // slices per tile
    uint32_t ring;   // shared address of the warp's two slice buffers
    uint32_t full;   // full[0]; full[1] = full + 8, empty[j] = full + 16 + 8 j
    uint32_t round;  // the warp's tile number
    __device__ __forceinline__ bool begin(uint32_t k) const {
        // BF16 slices 2 and 3 reuse the buffers of slices 0 and 1: wait for their MMAs (use u - 2);
        // the buffers of a tile's first two slices were freed before the tile started
        if (k % kSteps != 0 || k < 2u * kSteps) return true;
        const uint32_t u = kUses * round + k / kSteps;
        return mbar_wait(full + 16u + 8u * (u & 1u), ((u - 2u) >> 1) & 1u);
    }
    __device__ __forceinline__ void put(uint32_t k, uint32_t lane, Packer<DT> &pk) const {
        const uint32_t r = 32u * (k & 3u) + lane, slot = (k / kSteps) & 1u;
        uint32_t off;
        if constexpr (DT == EP_BF16)
            off = ((k >> 2) & 1u) * 128u;  // 16 bytes per step: chunk (k / 4) mod 2
        else
            off = ((k >> 3) & 1u) * 128u + ((k >> 2) & 1u) * 8u;  // 8 bytes per step
        pk.store_shared(ring + slot * kLinSlice + (r >> 3) * 256u + (r & 7u) * 16u + off);
    }
    __device__ __forceinline__ void end(uint32_t k, uint32_t lane) const {
        if (k % kSteps != kSteps - 1u) return;
        // the slice, written through the generic proxy, becomes visible to the tensor cores
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(full + 8u * ((k / kSteps) & 1u));
    }
};

// the X operand: BF16 (K = 16 per MMA) or the 8-bit codes of the quantized activations (K = 32);
// either way 32 bytes of a row per MMA, row n's 16-byte chunk c of a K tile at
// (n / 8) 8 XB + 128 c + 16 (n mod 8), XB the row's bytes per K tile
template <int DT>
struct XOperand {
    static constexpr uint32_t kRowBytes = DT == EP_BF16 ? 128u : 64u;  // one K tile (64 inputs) of a row
};

template <int DT, int MODE>
__global__ void __launch_bounds__((kLinMaxWarps + 1) * 32, 1) linear_kernel(const __grid_constant__ LinParams P) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr uint32_t XB = XOperand<DT>::kRowBytes;
    const Params &p = P.dp;
    constexpr uint32_t kTables = uint32_t(MODE == kPaired ? kPairedTableBytes : kLutBytes);
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5, S = P.S;
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const uint32_t lut = base;
    auto wbar = [&](uint32_t w) { return base + P.off_bars + kLinBarBytes * w; };  // full[2], empty[2], copy
    const uint32_t tbar = base + P.off_bars + kLinBarBytes * S, done = tbar + 8u, tmem_slot = tbar + 16u;
    auto ring = [&](uint32_t w) { return base + P.off_w + 2u * kLinSlice * w; };
    auto xbuf = [&](uint32_t w) { return base + P.off_x + P.npad * XB * w; };
    auto tbuf = [&](uint32_t w) { return base + P.off_tile + P.tile_buf * w; };
    const uint32_t band = blockIdx.x;
    const uint32_t kt0 = blockIdx.y * P.kt_per_split;
    const uint32_t nkt = min(P.KT, kt0 + P.kt_per_split) - kt0;  // >= 1: the plan leaves no split empty

    if (threadIdx.x == 0) {
        for (uint32_t w = 0; w < S; ++w)
            for (uint32_t i = 0; i < 5; ++i) mbar_init(wbar(w) + 8u * i, 1);
        mbar_init(tbar, 1);
        mbar_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_proxy_async();
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == S) {  // the accumulator's tensor memory (the whole warp allocates)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot),
                     "r"(P.tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (threadIdx.x == 0) {
        mbar_expect(tbar, kTables);
        bulk_g2s(lut, p.tables, kTables, tbar);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = lds32(tmem_slot);
    bool ok = mbar_wait(tbar, 0);
    uint32_t err = ok ? 0u : uint32_t(EP_DEC_TIMEOUT);

    if (warp < S) {
        // ---- decoding warps: tiles j = warp, warp + S, ... of the CTA's K range
        SliceSink<DT> sink{ring(warp), wbar(warp), 0u};
        const uint32_t copyb = wbar(warp) + 32u;
        for (uint32_t j = warp; j < nkt && ok; j += S, ++sink.round) {
            const uint32_t kt = kt0 + j, t = band * P.KT + kt;
            // the MMAs of the previous tile (its last slice, use U round - 1, in ring buffer 1, and
            // so all before it) are done: the X buffer and both slice buffers are free
            if (sink.round > 0 && !mbar_wait(wbar(warp) + 24u, ((SliceSink<DT>::kUses * sink.round - 1u) >> 1) & 1u)) {
                err |= EP_DEC_TIMEOUT;
                break;
            }
            const uint32_t beg = __ldg(p.dir + t), end = __ldg(p.dir + t + 1), bytes = (end - beg) * 16u;
            if (end < beg + uint32_t(kTileHead / 16) || uint64_t(end) > p.tile_units || bytes + kSlack > P.tile_buf) {
                err |= EP_DEC_BAD_TILE;
                break;
            }
            if (lane == 0) {
                fence_proxy_async();
                mbar_expect(copyb, bytes);
                bulk_g2s(tbuf(warp), p.tiles + size_t(beg) * 16, bytes, copyb);
            }
            // X rows n < npad, inputs 64 kt .. + 63 (zero for n >= M): XB / 16 lanes per row, 16 bytes
            // each (BF16 activations, or their 8-bit codes quantized by the launch before this one)
            constexpr uint32_t kLanesPerRow = XB / 16u;
            const uint32_t xb = xbuf(warp), c = lane % kLanesPerRow;
            const uint8_t *xrow = DT == EP_BF16 ? reinterpret_cast<const uint8_t *>(P.x) + 128u * kt : P.xq + 64u * kt;
            const size_t xstride = DT == EP_BF16 ? 2u * p.cols : p.cols;
            for (uint32_t n = lane / kLanesPerRow; n < P.npad; n += 32u / kLanesPerRow) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (n < P.M) v = __ldg(reinterpret_cast<const uint4 *>(xrow + size_t(n) * xstride) + c);
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(xb + (n >> 3) * 8u * XB + c * 128u +
                                                                              (n & 7u) * 16u),
                             "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                             : "memory");
            }
            if (!mbar_wait(copyb, sink.round & 1u)) {
                err |= EP_DEC_TIMEOUT;
                break;
            }
            const uint32_t e = decode_tile<DT, kRowsGemm, MODE, true, uint32_t, SliceSink<DT>>(
                p, lut, tbuf(warp), bytes, t, lane, &sink);
            err |= e;
            if (__any_sync(0xffffffffu, e != 0)) break;  // the tile's slices may be missing: stop here
        }
    } else if (warp == S) {
        // ---- the MMA issuer: round by round, slice by slice, warp by warp
        constexpr uint32_t U = SliceSink<DT>::kUses;
        const uint32_t rounds = (nkt + S - 1) / S;
        bool first = true;
        for (uint32_t r = 0; r < rounds && ok; ++r)
            for (uint32_t sl = 0; sl < U && ok; ++sl)
                for (uint32_t w = 0; w < S && r * S + w < nkt; ++w) {
                    const uint32_t u = U * r + sl, fb = wbar(w) + 8u * (u & 1u);
                    if (!mbar_wait(fb, (u >> 1) & 1u)) {
                        err |= EP_DEC_TIMEOUT;
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    if (lane == 0) {
                        const uint64_t da = umma_desc_plain(ring(w) + (u & 1u) * kLinSlice, 128u, 256u);
                        const uint64_t db = umma_desc_plain(xbuf(w) + 256u * sl, 128u, 8u * XB);
                        const uint32_t acc = first ? 0u : 1u;
                        if constexpr (DT == EP_BF16)
                            asm volatile(
                                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                                "l"(da), "l"(db), "r"(P.idesc), "r"(acc)
                                : "memory");
                        else if constexpr (DT == EP_INT8)
                            asm volatile(
                                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                                "l"(da), "l"(db), "r"(P.idesc), "r"(acc)
                                : "memory");
                        else
                            asm volatile(
                                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem),
                                "l"(da), "l"(db), "r"(P.idesc), "r"(acc)
                                : "memory");
                        asm volatile(
                            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                fb + 16u)
                            : "memory");
                    }
                    first = false;
                    __syncwarp();
                }
        if (lane == 0)
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(done)
                         : "memory");
        __syncwarp();
    }
    // ---- epilogue: warp q < 4 reads tensor-memory lanes 32 q .. 32 q + 31 (features), one column per
    // token, and writes each token's 32 features (128 contiguous bytes) of the partial sums
    if (warp < 4) {
        if (!mbar_wait(done, 0)) err |= EP_DEC_TIMEOUT;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        float *dst = P.part + size_t(blockIdx.y) * P.M * P.N + 128u * band + 32u * warp + lane;
        for (uint32_t c0 = 0; c0 < P.npad; c0 += 16u) {
            uint32_t r[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
                "%14, %15}, [%16];"
                : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                  "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                  "=r"(r[15])
                : "r"(tmem + ((32u * warp) << 16) + c0));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (uint32_t i = 0; i < 16u; ++i)  // fp32 sums, or the int32 sums of the INT8 MMA, as bits
                if (c0 + i < P.M) reinterpret_cast<uint32_t *>(dst)[size_t(c0 + i) * P.N] = r[i];
        }
    }
    if (err && p.status && lane == 0) atomicOr(p.status, err);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // the partial sums are visible device-wide before this CTA counts itself done
    __threadfence();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == S) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(P.tmem_cols)
                     : "memory");
    }
    // ---- the band's last CTA: Y = the splits' partial sums in split order, plus the bias
    if (threadIdx.x == 0) {
        const uint32_t ticket = atomicAdd(P.count + band, 1u);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(tmem_slot), "r"(ticket == P.splits - 1u ? 1u : 0u) : "memory");
    }
    __syncthreads();
    if (lds32(tmem_slot) == 0u) return;
    __threadfence();
    // four features per thread and step; the loads of up to eight splits are issued before their
    // additions, which stay in split order (INT8: exact int32 sums).  BF16: y = RNE(sum + bias).
    // Codes: y = RNE(fp32(fp32(sum) s_x) s_w), then with a bias RNE(y + bias): the order of the
    // per-row-quantized layers' own arithmetic
    using Acc = typename std::conditional<DT == EP_INT8, int32_t, float>::type;
    using Acc4 = typename std::conditional<DT == EP_INT8, int4, float4>::type;
    const size_t MN4 = size_t(P.M) * P.N / 4u;
    for (uint32_t i = threadIdx.x; i < P.M * 32u; i += blockDim.x) {
        const uint32_t m = i >> 5, n = 128u * band + 4u * (i & 31u);
        const Acc4 *src = reinterpret_cast<const Acc4 *>(P.part + size_t(m) * P.N + n);
        Acc a[4] = {Acc(0), Acc(0), Acc(0), Acc(0)};
        for (uint32_t s0 = 0; s0 < P.splits; s0 += 8u) {
            Acc4 v[8];
#pragma unroll
            for (uint32_t j = 0; j < 8u; ++j)
                if (s0 + j < P.splits) v[j] = __ldcg(src + (s0 + j) * MN4);
#pragma unroll
            for (uint32_t j = 0; j < 8u; ++j)
                if (s0 + j < P.splits) {
                    a[0] += v[j].x;
                    a[1] += v[j].y;
                    a[2] += v[j].z;
                    a[3] += v[j].w;
                }
        }
        uint16_t *dst = P.y + size_t(m) * P.N + n;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float yv;
            if constexpr (DT == EP_BF16) {
                yv = a[j];
                if (P.bias) yv += __uint_as_float(uint32_t(P.bias[n + j]) << 16);
            } else {
                const float f = DT == EP_INT8 ? __int2float_rn(int32_t(a[j])) : float(a[j]);
                yv = __fmul_rn(__fmul_rn(f, P.xscale[m]), __ldg(P.wscale + n + j));
                if (P.bias)
                    yv = __bfloat162float(__float2bfloat16_rn(yv)) + __uint_as_float(uint32_t(P.bias[n + j]) << 16);
            }
            const __nv_bfloat16 h = __float2bfloat16_rn(yv);
            dst[j] = *reinterpret_cast<const uint16_t *>(&h);
        }
    }
    if (threadIdx.x == 0) P.count[band] = 0u;  // ready for the next call
}

// The activations of a per-row-quantized layer: per token, scale = amax / 127 (INT8) or / 448 (FP8
// E4M3), 1 for an all-zero row; codes = x / scale rounded to nearest even and clamped to [-127, 127]
// (INT8), or clamped to [-448, 448] and rounded to E4M3 (FP8).  One CTA per token.
template <int DT>
__global__ void __launch_bounds__(256) quantize_x_kernel(const uint16_t *x, uint32_t K, uint8_t *xq, float *xscale) {
    __shared__ float part[8];
    const uint32_t m = blockIdx.x;
    const uint16_t *row = x + size_t(m) * K;
    float amax = 0.0f;
    for (uint32_t k = threadIdx.x; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(__uint_as_float(uint32_t(row[k]) << 16)));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, d));
    if ((threadIdx.x & 31u) == 0) part[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = part[0];
    for (uint32_t w = 1; w < (blockDim.x >> 5); ++w) amax = fmaxf(amax, part[w]);
    const float scale = amax > 0.0f ? __fdiv_rn(amax, DT == EP_INT8 ? 127.0f : 448.0f) : 1.0f;
    if (threadIdx.x == 0) xscale[m] = scale;
    uint8_t *out = xq + size_t(m) * K;
    for (uint32_t k = threadIdx.x; k < K; k += blockDim.x) {
        const float v = __fdiv_rn(__uint_as_float(uint32_t(row[k]) << 16), scale);
        if constexpr (DT == EP_INT8)
            out[k] = uint8_t(int8_t(__float2int_rn(fminf(fmaxf(rintf(v), -127.0f), 127.0f))));
        else
            out[k] = uint8_t(__nv_cvt_float_to_fp8(fminf(fmaxf(v, -448.0f), 448.0f), __NV_SATFINITE, __NV_E4M3));
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ host side
struct DeviceCache {
    std::mutex mu;
    int sms[64] = {0};
    bool attr[64][8] = {};
};
DeviceCache g_cache;

template <int DT>
cudaError_t launch(Params &p, uint64_t max_tile, int mode, bool gemm, int device, cudaStream_t stream) {
    int sms;
    {
        std::lock_guard<std::mutex> g(g_cache.mu);
        if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
        if (!g_cache.sms[device]) {
            cudaError_t e = cudaDeviceGetAttribute(&g_cache.sms[device], cudaDevAttrMultiProcessorCount, device);
            if (e != cudaSuccess) return e;
        }
        if (!g_cache.attr[device][DT]) {
            cudaError_t e = cudaSuccess;
            for (auto k : {decode_kernel<DT, kRowsAny, kNarrow>, decode_kernel<DT, kRows32, kNarrow>,
                           decode_kernel<DT, kRowsPadded, kNarrow>, decode_kernel<DT, kRowsGemm, kNarrow>,
                           decode_kernel<DT, kRowsAny, kWide>, decode_kernel<DT, kRows32, kWide>,
                           decode_kernel<DT, kRowsPadded, kWide>, decode_kernel<DT, kRowsGemm, kWide>,
                           decode_kernel<DT, kRowsAny, kPaired>, decode_kernel<DT, kRows32, kPaired>,
                           decode_kernel<DT, kRowsPadded, kPaired>, decode_kernel<DT, kRowsGemm, kPaired>})
                if (e == cudaSuccess)
                    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemLimit));
            if (e != cudaSuccess) return e;
            g_cache.attr[device][DT] = true;
        }
        sms = g_cache.sms[device];
    }
    // one CTA per SM (at most one per tile); warps = tiles per CTA, within kMaxWarps and the
    // tile buffers that fit beside the tables: two per warp when a warp has several tiles and
    // they fit, else one; when even one per warp does not fit, fewer warps with one buffer each
    // (the decode is bound by latency, so warps matter more than overlapping the next copy),
    // else the tiles are read from global memory
    uint32_t grid = p.T < uint32_t(sms) ? p.T : uint32_t(sms);
    uint32_t warps = (p.T + grid - 1) / grid;
    warps = warps > uint32_t(kMaxWarps) ? uint32_t(kMaxWarps) : warps;
    const size_t fixed = mode == kPaired ? kPairedFixedBytes : kFixedBytes;
    const size_t avail = kSmemLimit - fixed;
    p.tile_buf = uint32_t((max_tile + kSlack + 15) & ~uint64_t(15));
    bool many = p.T > grid * warps;  // some warp decodes more than one tile
    if (many && 2ull * warps * p.tile_buf <= avail) {
        p.nbuf = 2;
    } else if (uint64_t(warps) * p.tile_buf <= avail) {
        p.nbuf = 1;
    } else if (p.tile_buf <= avail) {
        warps = uint32_t(avail / p.tile_buf);
        p.nbuf = 1;
    } else {
        p.nbuf = 0;  // tiles beyond any buffer: read in place
        p.tile_buf = 16;
    }
    if (warps < 1) warps = 1;
    size_t smem = fixed + size_t(warps) * (p.nbuf ? p.nbuf : 1) * p.tile_buf;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(warps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (gemm) {
        if (mode == kPaired) return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsGemm, kPaired>, p);
        if (mode == kWide) return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsGemm, kWide>, p);
        return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsGemm, kNarrow>, p);
    }
    if (mode == kPaired) {
        if (p.cols & 7u) return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsPadded, kPaired>, p);
        if ((p.cb & 31u) == 0) return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRows32, kPaired>, p);
        return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsAny, kPaired>, p);
    }
    if (mode == kWide) {
        if (p.cols & 7u) return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsPadded, kWide>, p);
        if ((p.cb & 31u) == 0) return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRows32, kWide>, p);
        return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsAny, kWide>, p);
    }
    if (p.cols & 7u) return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsPadded, kNarrow>, p);
    if ((p.cb & 31u) == 0) return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRows32, kNarrow>, p);
    return cudaLaunchKernelEx(&cfg, decode_kernel<DT, kRowsAny, kNarrow>, p);
}

int check_info(const ep_info *info) {
    if (info->rows <= 0 || info->cols <= 0 || info->n_tiles == 0) return EP_ERR_INVALID_ARG;
    const int64_t cb = (info->cols + 7) / 8;  // rows zero-padded to whole E8 blocks
    if (info->rows >= (int64_t(1) << 31) || cb >= (int64_t(1) << 31) || info->rows * cb >= (int64_t(1) << 31))
        return EP_ERR_UNSUPPORTED;
    if (info->paired > 1) return EP_ERR_CORRUPT;
    if (info->layout > 1 || !layout_fits(int(info->layout), info->rows, info->cols, info->blocks_per_lane))
        return EP_ERR_CORRUPT;
    uint32_t total = 0;
    for (int c = 0; c < kContexts; ++c) {
        if (!split_valid(info->split[c], c) || info->ntok[c] > split_alphabet(info->split[c], kCtxLow[c]))
            return EP_ERR_CORRUPT;
        if (info->paired && info->split[c] > kCtxNarrowSplit[c]) return EP_ERR_CORRUPT;
        if (info->paired && (c == 1 || c == 2)) {
            if (info->ntok[c] > kPairMaxAlphabet) return EP_ERR_CORRUPT;
            total += pair_table_len(info->ntok[c]);
        } else {
            total += info->ntok[c];
        }
    }
    if (info->off_freq + 2ull * total > info->off_dir) return EP_ERR_CORRUPT;
    return EP_OK;
}

// the container's dtype, another float dtype for a float container, or the lattice points
bool out_dtype_ok(const ep_info *info, int32_t out_dtype) {
    auto is_float = [](int32_t d) { return d == EP_BF16 || d == EP_FP16 || d == EP_FP32; };
    return out_dtype == info->container_dtype || out_dtype == EP_LATTICE_I32 ||
           (is_float(out_dtype) && is_float(info->container_dtype));
}

// tables hold y = (v - c) / 2 instead of v for coordinates 1..7 when a split is beyond the
// narrow range (v itself would not fit the 9-bit value field)
bool wide_fields(const ep_info *info) {
    for (int c = 0; c < kContexts; ++c)
        if (info->split[c] > kCtxNarrowSplit[c]) return true;
    return false;
}

int coding_of(const ep_info *info) { return info->paired ? kPaired : wide_fields(info) ? kWide : kNarrow; }

uint32_t pack_splits(const ep_info *info) {
    uint32_t s = 0;
    for (int c = 0; c < kContexts; ++c) s |= uint32_t(info->split[c]) << (4 * c);
    return s;
}

// the decode kernels' view of a device stream and its prepared tables
Params params_of(const ep_info *info, const void *d_blob, const void *d_tables, void *d_out, uint32_t *d_status) {
    Params p;
    const uint8_t *base = static_cast<const uint8_t *>(d_blob);
    p.dir = reinterpret_cast<const uint32_t *>(base + info->off_dir);
    p.tiles = base + info->off_tiles;
    p.rowf = reinterpret_cast<const float *>(base + info->off_rowf);
    p.tables = static_cast<const uint32_t *>(d_tables);
    p.out = d_out;
    p.status = d_status;
    p.tile_units = (info->storage_nbytes - info->off_tiles) / 16;
    p.cols = uint64_t(info->cols);
    p.cb = uint32_t((info->cols + 7) / 8);
    p.nb = uint32_t(info->rows) * p.cb;
    p.rows = uint32_t(info->rows);
    p.K = info->blocks_per_lane;
    p.T = info->n_tiles;
    p.splits = pack_splits(info);
    for (int c = 0; c < 2; ++c) {
        p.pair_A[c] = info->paired ? info->ntok[1 + c] : 0u;
        p.pair_rawb[c] = pair_raw_bits(p.pair_A[c]);
    }
    p.tile_buf = 0;
    p.nbuf = 0;
    return p;
}

// ---- the fused GEMM's launch plan: bands of 128 output features, K tiles split across CTAs so that
// all CTAs run in one wave (one per SM); shared memory = tables, barriers, then per decoding warp a
// stream-tile buffer, two W slice buffers and an X buffer.  Decoding warps: as many as fit, then as
// few as give the same number of rounds of tiles.
struct LinPlan {
    uint32_t nbands, KT, splits, kt_per_split, S, npad, tmem_cols, tile_buf, off_bars, off_tile, off_w, off_x;
    uint32_t xrow;  // bytes of one token's K tile in the X buffer: 128 (BF16) or 64 (8-bit codes)
    bool codes;     // an INT8 / FP8 container: the activations are quantized per token first
    size_t smem;
};

LinPlan lin_plan(const ep_info *info, int sms, int64_t m) {
    LinPlan L{};
    L.nbands = uint32_t(info->rows / 128);
    L.KT = uint32_t(info->cols / 64);
    uint32_t splits_max = L.nbands < uint32_t(sms) ? uint32_t(sms) / L.nbands : 1u;
    splits_max = std::max(1u, std::min(splits_max, L.KT));
    L.kt_per_split = (L.KT + splits_max - 1) / splits_max;
    L.splits = (L.KT + L.kt_per_split - 1) / L.kt_per_split;
    L.npad = uint32_t((m + 15) / 16 * 16);
    L.codes = info->container_dtype != EP_BF16;
    L.xrow = L.codes ? 64u : 128u;
    L.tile_buf = uint32_t((info->max_tile_nbytes + kSlack + 15) & ~uint64_t(15));
    const uint32_t tables = uint32_t(info->paired ? kPairedTableBytes : kLutBytes);
    auto layout = [&](uint32_t S) {
        L.S = S;
        L.off_bars = tables;
        L.off_tile = (L.off_bars + kLinBarBytes * S + 24u + 15u) & ~15u;
        L.off_w = (L.off_tile + S * L.tile_buf + 127u) & ~127u;
        L.off_x = L.off_w + S * 2u * kLinSlice;
        L.smem = size_t(L.off_x) + size_t(S) * L.npad * L.xrow;
    };
    uint32_t S = std::min(kLinMaxWarps, L.kt_per_split);
    for (layout(S); S > 1 && L.smem > kSmemLimit; layout(--S)) {
    }
    const uint32_t rounds = (L.kt_per_split + S - 1) / S;
    layout((L.kt_per_split + rounds - 1) / rounds);
    L.tmem_cols = 32;
    while (L.tmem_cols < L.npad) L.tmem_cols *= 2;
    // more than half an SM's shared memory: one CTA per SM, so no CTA waits for another's tensor memory
    L.smem = std::max(L.smem, kSmemLimit / 2 + 1024);
    return L;
}

// the caller's scratch: the partial sums (splits x m x N, fp32 or int32), one counter per band, and
// for code containers the activations' codes (m x K bytes) and per-token scales (m floats)
size_t lin_count_offset(const LinPlan &L, int64_t m) {
    return (size_t(L.splits) * size_t(m) * size_t(L.nbands) * 128u * sizeof(float) + 15u) & ~size_t(15);
}
size_t lin_xq_offset(const LinPlan &L, int64_t m) {
    return (lin_count_offset(L, m) + size_t(L.nbands) * 4u + 15u) & ~size_t(15);
}
size_t lin_xscale_offset(const LinPlan &L, int64_t m) {
    return (lin_xq_offset(L, m) + size_t(m) * L.KT * 64u + 15u) & ~size_t(15);
}
size_t lin_work_bytes(const LinPlan &L, int64_t m) {
    return L.codes ? lin_xscale_offset(L, m) + size_t(m) * 4u : lin_count_offset(L, m) + size_t(L.nbands) * 4u;
}

}  // namespace
}  // namespace ep

extern "C" int ep_prepare(const ep_info *info, const void *d_blob, void *d_workspace, uint32_t *d_status,
                          ep_stream_t stream) {
    using namespace ep;
    if (!info || !d_blob || !d_workspace) return EP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_blob) | reinterpret_cast<uintptr_t>(d_workspace)) & 15u)
        return EP_ERR_INVALID_ARG;
    int rc = check_info(info);
    if (rc != EP_OK) return rc;
    PrepParams q;
    q.freq = reinterpret_cast<const uint16_t *>(static_cast<const uint8_t *>(d_blob) + info->off_freq);
    q.tables = static_cast<uint32_t *>(d_workspace);
    q.status = d_status;
    q.splits = pack_splits(info);
    q.wide = wide_fields(info) ? 1u : 0u;
    q.paired = info->paired ? 1u : 0u;
    q.tab_off[0] = 0;
    for (int c = 0; c < kContexts; ++c) {
        q.ntok[c] = info->ntok[c];
        const bool pair = info->paired && (c == 1 || c == 2);
        q.tab_off[c + 1] = q.tab_off[c] + (pair ? pair_table_len(info->ntok[c]) : info->ntok[c]);
    }
    const uint32_t grid = info->paired ? 5 * kPrepSingleCtas + 2 * kPrepPairCtas : kContexts * kPrepSingleCtas;
    prepare_kernel<<<grid, kPrepThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(q);
    return cudaGetLastError() == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

extern "C" int ep_decompress(const ep_info *info, const void *d_blob, const void *d_workspace, void *d_out,
                             int32_t out_dtype, uint32_t *d_status, ep_stream_t stream) {
    using namespace ep;
    if (!info || !d_blob || !d_workspace || !d_out) return EP_ERR_INVALID_ARG;
    if (!out_dtype_ok(info, out_dtype)) return EP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_blob) | reinterpret_cast<uintptr_t>(d_out) |
         reinterpret_cast<uintptr_t>(d_workspace)) & 15u)
        return EP_ERR_INVALID_ARG;
    int rc = check_info(info);
    if (rc != EP_OK) return rc;
    Params p = params_of(info, d_blob, d_workspace, d_out, d_status);
    int device;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) return EP_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint64_t mt = info->max_tile_nbytes;
    const int mode = coding_of(info);
    switch (out_dtype) {
    case EP_BF16: e = launch<EP_BF16>(p, mt, mode, info->layout == 1, device, s); break;
    case EP_FP16: e = launch<EP_FP16>(p, mt, mode, info->layout == 1, device, s); break;
    case EP_FP32: e = launch<EP_FP32>(p, mt, mode, info->layout == 1, device, s); break;
    case EP_INT8: e = launch<EP_INT8>(p, mt, mode, info->layout == 1, device, s); break;
    case EP_FP8_E4M3: e = launch<EP_FP8_E4M3>(p, mt, mode, info->layout == 1, device, s); break;
    case EP_LATTICE_I32: e = launch<EP_LATTICE_I32>(p, mt, mode, info->layout == 1, device, s); break;
    default: return EP_ERR_INVALID_ARG;
    }
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

// ------------------------------------------------------------------ ep_linear_fused
namespace ep {
namespace {

int device_sms(int *device, int *sms) {
    if (cudaGetDevice(device) != cudaSuccess || *device < 0 || *device >= 64) return EP_ERR_CUDA;
    std::lock_guard<std::mutex> g(g_cache.mu);
    if (!g_cache.sms[*device] &&
        cudaDeviceGetAttribute(&g_cache.sms[*device], cudaDevAttrMultiProcessorCount, *device) != cudaSuccess)
        return EP_ERR_CUDA;
    *sms = g_cache.sms[*device];
    return EP_OK;
}

bool linear_ok(const ep_info *info, int64_t m) {
    return info && info->layout == 1 &&
           (info->container_dtype == EP_BF16 || info->container_dtype == EP_INT8 ||
            info->container_dtype == EP_FP8_E4M3) &&
           m >= 1 && m <= 128 && check_info(info) == EP_OK;
}

struct LinCache {
    std::mutex mu;
    size_t smem_set[64][9] = {};  // [device][3 container + coding mode]
};
LinCache g_lin;

}  // namespace
}  // namespace ep

extern "C" size_t ep_linear_fused_workspace(const ep_info *info, int64_t m) {
    using namespace ep;
    if (!linear_ok(info, m)) return 0;
    int device, sms;
    if (device_sms(&device, &sms) != EP_OK) return 0;
    const LinPlan L = lin_plan(info, sms, m);
    return lin_work_bytes(L, m);
}

extern "C" int ep_linear_fused(const ep_info *info, const void *d_blob, const void *d_tables, const void *d_x,
                               int64_t m, const void *d_bias, void *d_y, void *d_work, size_t work_nbytes,
                               uint32_t *d_status, ep_stream_t stream) {
    using namespace ep;
    if (!d_blob || !d_tables || !d_x || !d_y || !d_work || !linear_ok(info, m)) return EP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_blob) | reinterpret_cast<uintptr_t>(d_tables) |
         reinterpret_cast<uintptr_t>(d_x) | reinterpret_cast<uintptr_t>(d_work)) & 15u)
        return EP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_y) & 1u || reinterpret_cast<uintptr_t>(d_bias) & 1u) return EP_ERR_INVALID_ARG;
    int device, sms;
    if (device_sms(&device, &sms) != EP_OK) return EP_ERR_CUDA;
    const LinPlan L = lin_plan(info, sms, m);
    if (work_nbytes < lin_work_bytes(L, m)) return EP_ERR_INVALID_ARG;
    if (L.smem > kSmemLimit) return EP_ERR_UNSUPPORTED;  // tiles too large for one warp's buffers beside the tables
    LinParams P;
    P.dp = params_of(info, d_blob, d_tables, nullptr, d_status);
    P.x = static_cast<const uint16_t *>(d_x);
    P.part = static_cast<float *>(d_work);
    P.count = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(d_work) + lin_count_offset(L, m));
    P.bias = static_cast<const uint16_t *>(d_bias);
    P.y = static_cast<uint16_t *>(d_y);
    P.splits = L.splits;
    P.M = uint32_t(m);
    P.N = uint32_t(info->rows);
    P.npad = L.npad;
    // the MMA's instruction descriptor: accumulator type (bits 4..5: 1 fp32, 2 int32), A and B types
    // (bits 7..9, 10..12: BF16 = 1 for kind::f16, signed = 1 for kind::i8, E4M3 = 0 for
    // kind::f8f6f4), both K-major, N = npad (bits 17..22: N / 8), M = 128 (bits 24..28: M / 16)
    const int dt = info->container_dtype;
    const uint32_t types = dt == EP_BF16 ? (1u << 4) | (1u << 7) | (1u << 10)
                           : dt == EP_INT8 ? (2u << 4) | (1u << 7) | (1u << 10)
                                           : (1u << 4);
    P.idesc = types | ((L.npad >> 3) << 17) | ((128u >> 4) << 24);
    P.tmem_cols = L.tmem_cols;
    P.KT = L.KT;
    P.kt_per_split = L.kt_per_split;
    P.S = L.S;
    P.tile_buf = L.tile_buf;
    P.off_bars = L.off_bars;
    P.off_tile = L.off_tile;
    P.off_w = L.off_w;
    P.off_x = L.off_x;
    uint8_t *work = static_cast<uint8_t *>(d_work);
    P.xq = L.codes ? work + lin_xq_offset(L, m) : nullptr;
    P.xscale = L.codes ? reinterpret_cast<const float *>(work + lin_xscale_offset(L, m)) : nullptr;
    P.wscale = L.codes ? reinterpret_cast<const float *>(static_cast<const uint8_t *>(d_blob) + info->off_scales)
                       : nullptr;
    const int mode = info->paired ? kPaired : (wide_fields(info) ? kWide : kNarrow);
    using Kern = void (*)(LinParams);
    // [container: BF16, INT8, FP8][coding mode]
    static const Kern kerns[3][3] = {
        {linear_kernel<EP_BF16, kNarrow>, linear_kernel<EP_BF16, kWide>, linear_kernel<EP_BF16, kPaired>},
        {linear_kernel<EP_INT8, kNarrow>, linear_kernel<EP_INT8, kWide>, linear_kernel<EP_INT8, kPaired>},
        {linear_kernel<EP_FP8_E4M3, kNarrow>, linear_kernel<EP_FP8_E4M3, kWide>, linear_kernel<EP_FP8_E4M3, kPaired>}};
    const int ci = dt == EP_BF16 ? 0 : (dt == EP_INT8 ? 1 : 2);
    const Kern kern = kerns[ci][mode];
    {
        std::lock_guard<std::mutex> g(g_lin.mu);
        size_t &set = g_lin.smem_set[device][3 * ci + mode];
        if (set < L.smem) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L.smem)) != cudaSuccess)
                return EP_ERR_CUDA;
            set = L.smem;
        }
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (L.codes) {  // the activations' codes and scales, into the scratch
        float *xs = reinterpret_cast<float *>(work + lin_xscale_offset(L, m));
        uint8_t *xq = work + lin_xq_offset(L, m);
        const uint16_t *x = static_cast<const uint16_t *>(d_x);
        if (dt == EP_INT8)
            quantize_x_kernel<EP_INT8><<<unsigned(m), 256, 0, s>>>(x, uint32_t(info->cols), xq, xs);
        else
            quantize_x_kernel<EP_FP8_E4M3><<<unsigned(m), 256, 0, s>>>(x, uint32_t(info->cols), xq, xs);
        if (cudaGetLastError() != cudaSuccess) return EP_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(L.nbands, L.splits);
    cfg.blockDim = dim3(std::max(L.S + 1, 4u) * 32);  // the epilogue needs warps 0..3
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, P) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

// ------------------------------------------------------------------ ep_decompress_noalloc
// The same decode for callers that cannot allocate device memory: the slot tables live in one
// file-scope device array instead of a caller workspace.  Every GPU that loads the library holds
// this array (106 KB) until the process exits; all calls on a device share it.
namespace ep {
namespace {

constexpr size_t kStaticTablesBytes = kPairedTableBytes;  // the largest workspace a stream can need
static __device__ __align__(256) uint32_t g_static_tables[kStaticTablesBytes / 4];

struct StaticTables {
    std::mutex mu;
    void *ptr[64] = {};
};
StaticTables g_static;

// device address of g_static_tables on the current device, looked up once per device (the host
// name of the array is only a stand-in and must not reach a kernel)
int static_tables(void **out) {
    int device;
    if (cudaGetDevice(&device) != cudaSuccess) return EP_ERR_CUDA;
    if (device < 0 || device >= 64) return EP_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> g(g_static.mu);
    if (!g_static.ptr[device]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_tables) != cudaSuccess || !p) return EP_ERR_CUDA;
        g_static.ptr[device] = p;
    }
    *out = g_static.ptr[device];
    return EP_OK;
}

}  // namespace
}  // namespace ep

extern "C" int ep_decompress_noalloc(const ep_info *info, const void *d_blob, void *d_out, int32_t out_dtype,
                                     uint32_t *d_status, ep_stream_t stream) {
    using namespace ep;
    if (!info || !d_blob || !d_out || !out_dtype_ok(info, out_dtype)) return EP_ERR_INVALID_ARG;
    if (info->workspace_nbytes > kStaticTablesBytes) return EP_ERR_UNSUPPORTED;
    void *tables = nullptr;
    int rc = static_tables(&tables);
    if (rc != EP_OK) return rc;
    // both launches go to the same stream, so the decode reads the tables this call prepared
    rc = ep_prepare(info, d_blob, tables, d_status, stream);
    if (rc != EP_OK) return rc;
    return ep_decompress(info, d_blob, tables, d_out, out_dtype, d_status, stream);
}

// ------------------------------------------------------------------ ep_decompress_host
// The same decode for a stream and an output in host memory: one copy in, ep_prepare,
// ep_decompress, one copy out, all on the caller's stream; the device buffers are carved from
// caller scratch (stream, tables, output, each 256-byte aligned).
namespace ep {
namespace {

size_t out_elt_bytes(int32_t dt) { return dt == EP_FP32 || dt == EP_LATTICE_I32 ? 4 : (dt == EP_BF16 || dt == EP_FP16) ? 2 : 1; }
size_t al256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace
}  // namespace ep

extern "C" size_t ep_decompress_host_scratch(const ep_info *info, int32_t out_dtype) {
    using namespace ep;
    if (!info || info->rows <= 0 || info->cols <= 0 || !out_dtype_ok(info, out_dtype)) return 0;
    return al256(info->storage_nbytes) + al256(info->workspace_nbytes) +
           al256(size_t(info->rows) * size_t(info->cols) * out_elt_bytes(out_dtype));
}

extern "C" int ep_decompress_host(const ep_info *info, const void *h_blob, void *h_out, int32_t out_dtype,
                                  void *d_scratch, size_t scratch_nbytes, uint32_t *d_status, ep_stream_t stream) {
    using namespace ep;
    if (!info || !h_blob || !h_out || !d_scratch || !out_dtype_ok(info, out_dtype)) return EP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(d_scratch) & 255u) return EP_ERR_INVALID_ARG;
    int rc = check_info(info);
    if (rc != EP_OK) return rc;
    if (scratch_nbytes < ep_decompress_host_scratch(info, out_dtype)) return EP_ERR_INVALID_ARG;
    uint8_t *d_blob = static_cast<uint8_t *>(d_scratch);
    uint8_t *d_work = d_blob + al256(info->storage_nbytes);
    uint8_t *d_out = d_work + al256(info->workspace_nbytes);
    const size_t out_bytes = size_t(info->rows) * size_t(info->cols) * out_elt_bytes(out_dtype);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(d_blob, h_blob, info->storage_nbytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return EP_ERR_CUDA;
    rc = ep_prepare(info, d_blob, d_work, d_status, stream);
    if (rc != EP_OK) return rc;
    rc = ep_decompress(info, d_blob, d_work, d_out, out_dtype, d_status, stream);
    if (rc != EP_OK) return rc;
    return cudaMemcpyAsync(h_out, d_out, out_bytes, cudaMemcpyDeviceToHost, s) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
