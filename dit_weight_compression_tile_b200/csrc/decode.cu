// Fused tile decode for sm_100a: ep_decompress.
//
// "The final coordinates are entropy-coded in independently decodable tiles, enabling fast,
// fused symbol decoding and numerical weight reconstruction on the GPU" ("EntroPack: Fast and
// Accurate Entropy-Coded Weight Compression at Arbitrary Bitrates", Abstract).  One kernel:
//   * each CTA turns the stream's frequency tables into seven 2048-slot tables in shared
//     memory; a slot's 32-bit entry holds the symbol's frequency, the slot's offset inside the
//     symbol, an escape flag and, for direct tokens, the decoded signed coordinate value;
//   * each warp decodes whole tiles: the tile is staged into the warp's shared-memory buffer
//     with 16-byte async copies, and lane l runs the rANS coder of lane l over its own word
//     stream, so a step needs no warp-wide exchange and its word address is known before the
//     state update that decides whether to consume it;
//   * the 8 coordinates of a lane's block are rebuilt in registers (coset from coordinate 0,
//     parity-forced coordinate 7), scaled by the row factor with one fp32 multiply and
//     converted to the container (BF16 / FP16 / FP32 / INT8 / FP8-E4M3) with round to nearest
//     even; a warp writes 32 consecutive blocks with one 16-byte (8-byte for codes) store per
//     lane.
// The path is a scan over compressed bytes, bound by HBM bandwidth and instruction issue; it
// uses no tensor cores because nothing in it is a dense contraction.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/eptile.h"
#include "format.h"

namespace ep {
namespace {

constexpr int kMaxWarps = 32;
constexpr uint32_t kLutEntries = kContexts * kProbScale;
constexpr uint32_t kTileBufMax = 16384;  // largest per-warp tile buffer; larger tiles are read in place
constexpr size_t kSmemLimit = 232448;    // shared memory one CTA may use on sm_100
constexpr size_t kLutBytes = size_t(kLutEntries) * 4;
constexpr size_t kTinfoBytes = size_t(kContexts) * 256 * 4;
constexpr size_t kCumBytes = (size_t(kContexts) * 257 * 4 + 15) & ~size_t(15);  // keeps the tile buffers 16-byte aligned
constexpr size_t kFixedBytes = kLutBytes + kTinfoBytes + kCumBytes;
static_assert(kFixedBytes % 16 == 0, "tile buffers must start 16-byte aligned");
constexpr size_t smem_bytes(uint32_t warps, uint32_t tile_buf) { return kFixedBytes + size_t(warps) * tile_buf; }

// slot entry: bias [0,11) | value or token [11,19) | escape [19] | frequency [20,32)
constexpr uint32_t kEsc = 1u << 19;

struct Params {
    const uint32_t *dir;     // tile directory, 16-byte units (T + 1 entries)
    const uint8_t *tiles;    // tile section
    const float *rowf;       // per-row factors f_r
    const uint16_t *freq;    // frequency tables, contexts in order
    void *out;               // container, row-major
    uint32_t *status;        // nullable
    uint64_t tile_units;     // size of the tile section in 16-byte units
    uint32_t nb;             // E8 blocks (rows * cols / 8)
    uint32_t cb;             // blocks per row
    uint32_t K;              // blocks per lane
    uint32_t T;              // tiles
    uint32_t tile_buf;       // bytes of each warp's tile buffer (multiple of 16)
    uint32_t splits;         // 3 bits per context
    uint32_t tab_off[kContexts + 1];  // table start of each context (prefix sum of ntok)
};

// ------------------------------------------------------------------ containers
template <int DT>
struct Packer;

__device__ __forceinline__ float reconstruct(int32_t v, float fr) { return __fmul_rn(fr, __int2float_rn(v)); }

template <>
struct Packer<EP_BF16> {
    uint32_t o[4];
    float lo;
    __device__ __forceinline__ void put(int i, int32_t v, float fr) {
        float w = reconstruct(v, fr);
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
};

template <>
struct Packer<EP_FP16> {
    uint32_t o[4];
    float lo;
    __device__ __forceinline__ void put(int i, int32_t v, float fr) {
        float w = reconstruct(v, fr);
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
};

template <>
struct Packer<EP_FP32> {
    float o[8];
    __device__ __forceinline__ void put(int i, int32_t v, float fr) { o[i] = reconstruct(v, fr); }
    __device__ __forceinline__ void store(void *out, uint32_t b) {
        float4 *p = reinterpret_cast<float4 *>(out) + 2 * size_t(b);
        p[0] = make_float4(o[0], o[1], o[2], o[3]);
        p[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
};

template <>
struct Packer<EP_INT8> {
    uint32_t o[2];
    __device__ __forceinline__ void put(int i, int32_t v, float fr) {
        int q = min(127, max(-127, __float2int_rn(reconstruct(v, fr))));
        uint32_t byte = uint32_t(q) & 0xffu;
        if ((i & 3) == 0)
            o[i >> 2] = byte;
        else
            o[i >> 2] |= byte << (8 * (i & 3));
    }
    __device__ __forceinline__ void store(void *out, uint32_t b) {
        reinterpret_cast<uint2 *>(out)[b] = make_uint2(o[0], o[1]);
    }
};

template <>
struct Packer<EP_FP8_E4M3> {
    uint32_t o[2];
    float lo;
    __device__ __forceinline__ void put(int i, int32_t v, float fr) {
        float w = reconstruct(v, fr);
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
};

// the lattice points themselves (v = 2z, int32), for consumers and bit-exact checks
template <>
struct Packer<EP_LATTICE_I32> {
    int32_t o[8];
    __device__ __forceinline__ void put(int i, int32_t v, float) { o[i] = v; }
    __device__ __forceinline__ void store(void *out, uint32_t b) {
        int4 *p = reinterpret_cast<int4 *>(out) + 2 * size_t(b);
        p[0] = make_int4(o[0], o[1], o[2], o[3]);
        p[1] = make_int4(o[4], o[5], o[6], o[7]);
    }
};

// ------------------------------------------------------------------ async copies (16 B per lane)
__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_dst), "l"(gsrc) : "memory");
}

// ------------------------------------------------------------------ a lane's word stream
// The tile's words live either in the warp's shared-memory buffer (SMEM) or, for a tile larger
// than the buffer, in global memory.  Indices are clamped to the tile's last word, so a damaged
// stream can only read inside its own tile.
template <bool SMEM>
struct Words;

template <>
struct Words<true> {
    uint32_t base;  // shared-memory address of word 0
    __device__ __forceinline__ uint32_t at(uint32_t i) const {
        uint32_t w;
        asm volatile("ld.shared.u16 %0, [%1];" : "=r"(w) : "r"(base + 2u * i));
        return w;
    }
};

template <>
struct Words<false> {
    const uint16_t *base;
    __device__ __forceinline__ uint32_t at(uint32_t i) const { return __ldg(base + i); }
};

struct Lane {
    uint32_t x;     // rANS state
    uint32_t idx;   // index (in the tile's word area) of the next word this lane would read
    uint32_t last;  // last word index of the tile
    uint32_t w;     // that word, fetched as soon as the previous one was consumed
};

__device__ __forceinline__ int32_t unzigzag(uint32_t u) { return int32_t(u >> 1) ^ -int32_t(u & 1u); }

// One coordinate of one lane: a rANS step through the context's slot table.  The word the
// lane would read is fetched before the state update so the load overlaps the table lookup.
// An escape token (rare: the token split keeps 99.9% of values direct) is followed by chunks of
// raw extra bits, at most 11 bits each, least significant first, each a uniform symbol taking
// the top bits of the slot; the warp runs them together, masked per lane.
template <bool SMEM, bool ACT>
__device__ __forceinline__ int32_t step(Lane &s, bool act, const uint32_t *lut, const uint32_t *tinfo,
                                        const Words<SMEM> &W) {
    uint32_t e = lut[s.x & (kProbScale - 1)];
    uint32_t x = (e >> 20) * (s.x >> kProbBits) + (e & 0x7ffu);
    bool need = x < kStateLow && (!ACT || act);
    if (need) {
        x = __byte_perm(s.w, x, 0x5410);  // (x << 16) | w for x < 2^16
        s.w = W.at(min(++s.idx, s.last));
    }
    if (!ACT || act) s.x = x;
    int32_t val = int32_t(e << 13) >> 24;  // bits [11, 19): the signed value of a direct token
    bool esc = (e & kEsc) && (!ACT || act);
    if (__any_sync(0xffffffffu, esc)) {
        uint32_t ti = esc ? tinfo[(e >> 11) & 0xffu] : 0u;  // (value base << 5) | raw extra bits
        uint32_t u = ti >> 5, nbits = ti & 31u, shift = 0;
#pragma unroll 1
        for (int j = 0; j < 2 && __any_sync(0xffffffffu, nbits != 0); ++j) {
            if (nbits != 0) {
                uint32_t bits = nbits < kChunkBits ? nbits : kChunkBits;
                uint32_t keep = kProbBits - bits;
                uint32_t slot = s.x & (kProbScale - 1);
                uint32_t xc = ((s.x >> kProbBits) << keep) | (slot & ((1u << keep) - 1u));
                if (xc < kStateLow) {
                    xc = __byte_perm(s.w, xc, 0x5410);
                    s.w = W.at(min(++s.idx, s.last));
                }
                u |= (slot >> keep) << shift;
                s.x = xc;
                shift += bits;
                nbits -= bits;
            }
        }
        if (esc) val = unzigzag(u);
    }
    return val;
}

// ------------------------------------------------------------------ one tile
template <int DT, bool SMEM, bool ACT>
__device__ __forceinline__ void decode_blocks(const Params &p, Lane &s, const uint32_t *lut, const uint32_t *tinfo,
                                              const Words<SMEM> &W, uint32_t t, uint32_t lane) {
    uint32_t b = t * 32u * p.K + lane;
    uint32_t row = b / p.cb, col = b - row * p.cb;
    float fr = b < p.nb ? __ldg(p.rowf + row) : 0.0f;  // row factor, loaded one block ahead
    for (uint32_t k = 0; k < p.K; ++k, b += 32u) {
        if (ACT && b - lane >= p.nb) break;
        bool act = !ACT || b < p.nb;
        uint32_t col_n = col + 32u, row_n = row;
        while (col_n >= p.cb) {
            col_n -= p.cb;
            ++row_n;
        }
        float fr_n = (k + 1 < p.K && b + 32u < p.nb) ? __ldg(p.rowf + row_n) : 0.0f;
        Packer<DT> pk;
        // coordinate 0 carries the coset c = v0 mod 2; y0 = floor(v0 / 2)
        int32_t v = step<SMEM, ACT>(s, act, lut, tinfo, W);
        int32_t c = v & 1;
        int32_t par = v >> 1;
        pk.put(0, v, fr);
        const uint32_t *lb = lut + (1u + uint32_t(c)) * kProbScale;
        const uint32_t *tb = tinfo + (1u + uint32_t(c)) * 256u;
#pragma unroll
        for (int i = 1; i < 7; ++i) {
            int32_t y = step<SMEM, ACT>(s, act, lb, tb, W);
            par ^= y;
            pk.put(i, 2 * y + c, fr);
        }
        // coordinate 7: E8 forces y7 = y0 + ... + y6 (mod 2)
        par &= 1;
        uint32_t c7 = 3u + 2u * uint32_t(c) + uint32_t(par);
        int32_t t7 = step<SMEM, ACT>(s, act, lut + c7 * kProbScale, tinfo + c7 * 256u, W);
        pk.put(7, 2 * (2 * t7 + par) + c, fr);
        if (act) pk.store(p.out, b);
        col = col_n;
        row = row_n;
        fr = fr_n;
    }
}

// Decodes tile t with one warp.  Returns the EP_DEC_* bits of this lane.
template <int DT, bool SMEM>
__device__ __forceinline__ uint32_t decode_tile(const Params &p, const uint32_t *lut, const uint32_t *tinfo,
                                                const uint8_t *head, const Words<SMEM> &W, uint32_t tile_bytes,
                                                uint32_t t, uint32_t lane) {
    // the 32 initial states and word counts; each lane's stream starts after the lower lanes'
    Lane s;
    uint32_t n;
    if (SMEM) {
        uint32_t h = static_cast<uint32_t>(__cvta_generic_to_shared(head));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(s.x) : "r"(h + 4u * lane));
        asm volatile("ld.shared.u16 %0, [%1];" : "=r"(n) : "r"(h + 128u + 2u * lane));
    } else {
        s.x = __ldg(reinterpret_cast<const uint32_t *>(head) + lane);
        n = __ldg(reinterpret_cast<const uint16_t *>(head + 128) + lane);
    }
    uint32_t incl = n;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= uint32_t(d)) incl += y;
    }
    uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t capacity = (tile_bytes - uint32_t(kTileHead)) / 2u;
    if (total > capacity) return EP_DEC_WORD_OVERRUN;  // warp-uniform: the counts overrun the tile
    uint32_t start = incl - n;
    s.idx = start;
    s.last = capacity ? capacity - 1u : 0u;
    s.w = W.at(min(s.idx, s.last));
    if (uint64_t(t + 1) * 32u * p.K <= p.nb)
        decode_blocks<DT, SMEM, false>(p, s, lut, tinfo, W, t, lane);
    else
        decode_blocks<DT, SMEM, true>(p, s, lut, tinfo, W, t, lane);
    uint32_t err = 0;
    if (s.x != kStateLow) err |= EP_DEC_BAD_END;
    uint32_t used = s.idx - start;
    if (used != n) err |= used > n ? EP_DEC_WORD_OVERRUN : EP_DEC_WORD_COUNT;
    if (capacity - total >= 8u) err |= EP_DEC_WORD_COUNT;
    return err;
}

// ------------------------------------------------------------------ kernel
template <int DT>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) decode_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(16) uint32_t smem[];
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    uint32_t *lut = smem;                                            // [ctx][slot]
    uint32_t *tinfo = smem + kLutEntries;                            // [ctx][token]
    uint32_t *cum = tinfo + kContexts * 256;                         // [ctx][257]
    uint8_t *buf = reinterpret_cast<uint8_t *>(smem) + kFixedBytes + size_t(warp) * p.tile_buf;

    // ---- this warp's first tile starts loading now, behind the table set-up
    uint32_t t_begin = uint32_t(uint64_t(blockIdx.x) * p.T / gridDim.x);
    uint32_t t_end = uint32_t(uint64_t(blockIdx.x + 1) * p.T / gridDim.x);
    const uint32_t buf_s = static_cast<uint32_t>(__cvta_generic_to_shared(buf));
    auto stage = [&](uint32_t t) {  // tile t into the buffer if it is valid and fits; no wait
        uint32_t beg = __ldg(p.dir + t), end = __ldg(p.dir + t + 1);
        if (end >= beg + uint32_t(kTileHead / 16) && uint64_t(end) <= p.tile_units && (end - beg) * 16u <= p.tile_buf) {
            const uint8_t *tp = p.tiles + size_t(beg) * 16;
            for (uint32_t i = lane; i < end - beg; i += 32u) cp_async16(buf_s + 16u * i, tp + 16u * i);
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
    if (t_begin + warp < t_end) stage(t_begin + warp);

    // ---- tables.  Every slot starts as an escape to token 255 with f = 2^11 and bias = slot
    // (an identity step that decodes nothing: a damaged stream then fails its end checks);
    // token info starts at zero.  Then the cumulative frequencies per context (warps take
    // contexts round robin), then the slots of every token.
    for (uint32_t i = threadIdx.x; i < kLutEntries; i += blockDim.x)
        lut[i] = (kProbScale << 20) | kEsc | (255u << 11) | (i & (kProbScale - 1));
    for (uint32_t i = threadIdx.x; i < kContexts * 256u; i += blockDim.x) tinfo[i] = 0;
    for (uint32_t c = warp; c < uint32_t(kContexts); c += nwarps) {
        uint32_t n = p.tab_off[c + 1] - p.tab_off[c], run = 0;
        for (uint32_t base = 0; base < n; base += 32) {
            uint32_t t = base + lane;
            uint32_t f = t < n ? uint32_t(p.freq[p.tab_off[c] + t]) : 0u;
            uint32_t incl = f;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= uint32_t(d)) incl += y;
            }
            if (t < n) cum[c * 257 + t] = run + incl - f;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            cum[c * 257 + n] = run;
            if (n && run != kProbScale && p.status) atomicOr(p.status, EP_DEC_BAD_TOKEN);
        }
    }
    __syncthreads();
    for (uint32_t i = warp; i < p.tab_off[kContexts]; i += nwarps) {
        uint32_t c = 0;
        while (c + 1 < uint32_t(kContexts) && p.tab_off[c + 1] <= i) ++c;
        uint32_t t = i - p.tab_off[c];
        uint32_t m = (p.splits >> (3 * c)) & 7u;
        bool esc = t >= (1u << m);
        // a direct token's value is unzigzag(token); an escape keeps the token index
        uint32_t field = esc ? t : (uint32_t(unzigzag(t)) & 0xffu);
        uint32_t lo = cum[c * 257 + t], f = cum[c * 257 + t + 1] - lo;
        uint32_t fill = f < kProbScale ? f : kProbScale;
        uint32_t head = (fill << 20) | (esc ? kEsc : 0u) | (field << 11);
        for (uint32_t sl = lane; sl < fill; sl += 32)
            if (lo + sl < kProbScale) lut[c * kProbScale + lo + sl] = head | sl;
        if (lane == 0 && esc) {
            // token -> value base and raw extra bits (h = min(m, 2))
            uint32_t h = m < 2 ? m : 2;
            uint32_t d = t - (1u << m), nn = m + (d >> h);
            uint32_t nbits = nn - h;
            uint32_t base = ((1u << h) | (d & ((1u << h) - 1u))) << (nbits & 31u);
            tinfo[c * 256 + t] = nbits <= 21 ? (base << 5) | nbits : 0u;
        }
    }
    __syncthreads();

    // ---- tiles of this CTA: a contiguous range, warps round robin
    for (uint32_t t = t_begin + warp; t < t_end; t += nwarps) {
        if (t != t_begin + warp) {
            __syncwarp();  // the previous tile's reads of the buffer are done
            stage(t);
        }
        uint32_t beg = __ldg(p.dir + t), end = __ldg(p.dir + t + 1);
        uint32_t err;
        if (end < beg + uint32_t(kTileHead / 16) || uint64_t(end) > p.tile_units) {
            err = EP_DEC_BAD_TILE;
        } else {
            const uint8_t *tp = p.tiles + size_t(beg) * 16;
            uint32_t tile_bytes = (end - beg) * 16u;
            if (tile_bytes <= p.tile_buf) {
                asm volatile("cp.async.wait_all;\n" ::: "memory");
                __syncwarp();
                Words<true> W{buf_s + uint32_t(kTileHead)};
                err = decode_tile<DT, true>(p, lut, tinfo, buf, W, tile_bytes, t, lane);
            } else {
                Words<false> W{reinterpret_cast<const uint16_t *>(tp + kTileHead)};
                err = decode_tile<DT, false>(p, lut, tinfo, tp, W, tile_bytes, t, lane);
            }
        }
        if (err && p.status) atomicOr(p.status, err);
    }
}

// ------------------------------------------------------------------ host side
struct DeviceCache {
    std::mutex mu;
    int sms[64] = {0};
    bool attr[64][8] = {};
};
DeviceCache g_cache;

template <int DT>
cudaError_t launch(const Params &p, int device, cudaStream_t stream) {
    int sms;
    {
        std::lock_guard<std::mutex> g(g_cache.mu);
        if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
        if (!g_cache.sms[device]) {
            cudaError_t e = cudaDeviceGetAttribute(&g_cache.sms[device], cudaDevAttrMultiProcessorCount, device);
            if (e != cudaSuccess) return e;
        }
        if (!g_cache.attr[device][DT]) {
            cudaError_t e = cudaFuncSetAttribute(decode_kernel<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 int(kSmemLimit));
            if (e != cudaSuccess) return e;
            g_cache.attr[device][DT] = true;
        }
        sms = g_cache.sms[device];
    }
    // one CTA per SM, as many warps as tiles per SM, at most kMaxWarps and as many tile buffers
    // as fit beside the tables
    uint32_t cap = uint32_t((kSmemLimit - kFixedBytes) / p.tile_buf);
    uint32_t warps = (p.T + uint32_t(sms) - 1) / uint32_t(sms);
    warps = warps < 1 ? 1 : warps;
    warps = warps > uint32_t(kMaxWarps) ? uint32_t(kMaxWarps) : warps;
    warps = warps > cap ? cap : warps;
    uint32_t grid = (p.T + warps - 1) / warps;
    if (grid > uint32_t(sms)) grid = uint32_t(sms);
    decode_kernel<DT><<<grid, warps * 32, smem_bytes(warps, p.tile_buf), stream>>>(p);
    return cudaGetLastError();
}

}  // namespace
}  // namespace ep

extern "C" int ep_decompress(const ep_info *info, const void *d_blob, void *d_out, int32_t out_dtype,
                             uint32_t *d_status, ep_stream_t stream) {
    using namespace ep;
    if (!info || !d_blob || !d_out) return EP_ERR_INVALID_ARG;
    if (out_dtype != info->container_dtype && out_dtype != EP_LATTICE_I32) return EP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_blob) | reinterpret_cast<uintptr_t>(d_out)) & 15u) return EP_ERR_INVALID_ARG;
    if (info->rows <= 0 || info->cols <= 0 || info->cols % 8 || info->n_tiles == 0) return EP_ERR_INVALID_ARG;
    int64_t nb = info->rows * (info->cols / 8);
    if (nb >= (int64_t(1) << 31) || info->cols / 8 >= (int64_t(1) << 31)) return EP_ERR_UNSUPPORTED;
    Params p;
    const uint8_t *base = static_cast<const uint8_t *>(d_blob);
    p.dir = reinterpret_cast<const uint32_t *>(base + info->off_dir);
    p.tiles = base + info->off_tiles;
    p.rowf = reinterpret_cast<const float *>(base + info->off_rowf);
    p.freq = reinterpret_cast<const uint16_t *>(base + info->off_freq);
    p.out = d_out;
    p.status = d_status;
    p.tile_units = (info->storage_nbytes - info->off_tiles) / 16;
    p.nb = uint32_t(nb);
    p.cb = uint32_t(info->cols / 8);
    p.K = info->blocks_per_lane;
    p.T = info->n_tiles;
    {
        uint64_t need = (info->max_tile_nbytes + 15) & ~uint64_t(15);
        // at least one 16-byte piece past the tile head, so a clamped word read stays inside
        p.tile_buf = uint32_t(need < kTileHead + 16 ? kTileHead + 16 : (need > kTileBufMax ? kTileBufMax : need));
    }
    p.splits = 0;
    p.tab_off[0] = 0;
    for (int c = 0; c < kContexts; ++c) {
        if (info->split[c] > kMaxSplit || info->ntok[c] > 256) return EP_ERR_CORRUPT;
        p.splits |= uint32_t(info->split[c]) << (3 * c);
        p.tab_off[c + 1] = p.tab_off[c] + info->ntok[c];
    }
    int device;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) return EP_ERR_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (out_dtype) {
    case EP_BF16: e = launch<EP_BF16>(p, device, s); break;
    case EP_FP16: e = launch<EP_FP16>(p, device, s); break;
    case EP_FP32: e = launch<EP_FP32>(p, device, s); break;
    case EP_INT8: e = launch<EP_INT8>(p, device, s); break;
    case EP_FP8_E4M3: e = launch<EP_FP8_E4M3>(p, device, s); break;
    case EP_LATTICE_I32: e = launch<EP_LATTICE_I32>(p, device, s); break;
    default: return EP_ERR_INVALID_ARG;
    }
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
