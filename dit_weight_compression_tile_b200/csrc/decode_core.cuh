// The decode's shared core (decode.cu: ep_decompress; linear.cu: ep_linear_fused): the stream's
// launch parameters, the container packers, a lane's rANS steps over its word region, the escape
// paths and the block loop of one tile ("EntroPack: Fast and Accurate Entropy-Coded Weight
// Compression at Arbitrary Bitrates", Abstract: tiles that decode on their own, decoded together
// with the weights' reconstruction), plus the host checks that turn an ep_info into parameters.
// Everything sits in an unnamed namespace: each kernel file gets its own copy.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>

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
    // the 8 values as 16 bytes at a shared-memory address (an operand slice of the fused GEMM)
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
        // GEMM-ordered tiles: four steps per unrolled iteration, so that the step's row of the
        // group of four (its factor, its place in the operand slice) is known when compiled
#pragma unroll (GEMM ? 4 : 1)
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

// ------------------------------------------------------------------ host checks and parameters
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

}  // namespace
}  // namespace ep
