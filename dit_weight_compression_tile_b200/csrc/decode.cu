// Fused tile decode for sm_100a: ep_decompress.
//
// "The final coordinates are entropy-coded in independently decodable tiles, enabling fast,
// fused symbol decoding and numerical weight reconstruction on the GPU" ("EntroPack: Fast and
// Accurate Entropy-Coded Weight Compression at Arbitrary Bitrates", Abstract).  One kernel:
//   * each CTA builds the seven slot -> (token, frequency, offset) tables of the stream in
//     shared memory (57 KB) from the stream's frequency tables;
//   * each warp decodes whole tiles: lane l is the rANS state of lane l, a step decodes one
//     symbol per lane, and renormalisation is warp-cooperative (ballot + popc gives each lane
//     its word index in the tile's 16-bit word stream);
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
constexpr size_t kSmemBytes = kLutEntries * 4 + kContexts * 257 * 4;

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

// ------------------------------------------------------------------ rANS lanes
struct Lane {
    uint32_t x;             // rANS state
    uint32_t pos;           // words consumed by the warp (warp-uniform)
    uint32_t err;           // EP_DEC_* bits
    uint32_t nwords;        // words in the tile
    uint32_t lt;            // lanes below this one
    const uint16_t *words;  // the tile's word stream
};

// lanes that fell below 2^16 read one word each, lower lanes first
__device__ __forceinline__ void renormalise(Lane &s, bool need) {
    uint32_t mask = __ballot_sync(0xffffffffu, need);
    if (need) {
        uint32_t idx = s.pos + __popc(mask & s.lt);
        uint32_t w = 0;
        if (idx < s.nwords)
            w = __ldg(s.words + idx);
        else
            s.err |= EP_DEC_WORD_OVERRUN;
        s.x = (s.x << 16) | w;
    }
    s.pos += __popc(mask);
}

// One coordinate: a token step through the context table, then the chunk steps of its raw
// extra bits.  Returns the zigzag value u.  All 32 lanes must call it.
__device__ __forceinline__ uint32_t decode_value(Lane &s, bool act, const uint32_t *lut, uint32_t m) {
    uint32_t e = lut[s.x & (kProbScale - 1)];
    uint32_t f = (e >> 12) & 0xfffu, bias = e & 0xfffu, tok = e >> 24;
    if (act) s.x = f * (s.x >> kProbBits) + bias;
    renormalise(s, act && s.x < kStateLow);
    uint32_t lim = 1u << m;
    uint32_t u = tok, nbits = 0;
    if (tok >= lim) {
        uint32_t h = m < 2 ? m : 2;
        uint32_t d = tok - lim;
        uint32_t n = m + (d >> h);
        nbits = n - h;
        if (nbits > 21) {  // no valid stream gets here: values stay below 2^22
            nbits = 0;
            s.err |= EP_DEC_BAD_TOKEN;
        }
        u = ((1u << h) | (d & ((1u << h) - 1u))) << nbits;
    }
    if (!act) nbits = 0;
    if (__any_sync(0xffffffffu, nbits != 0)) {
        uint32_t shift = 0;
#pragma unroll 1
        for (int j = 0; j < 2; ++j) {
            bool a = nbits != 0;
            if (!__any_sync(0xffffffffu, a)) break;
            if (a) {
                uint32_t b = nbits < kChunkBits ? nbits : kChunkBits;
                uint32_t keep = kProbBits - b;  // the chunk is the top b bits of the slot
                uint32_t slot = s.x & (kProbScale - 1);
                u |= (slot >> keep) << shift;
                s.x = ((s.x >> kProbBits) << keep) | (slot & ((1u << keep) - 1u));
                shift += b;
                nbits -= b;
            }
            renormalise(s, a && s.x < kStateLow);
        }
    }
    return u;
}

__device__ __forceinline__ int32_t unzigzag(uint32_t u) { return int32_t(u >> 1) ^ -int32_t(u & 1u); }

__device__ __forceinline__ uint32_t split_of(uint32_t splits, uint32_t ctx) { return (splits >> (3 * ctx)) & 7u; }

// ------------------------------------------------------------------ kernel
template <int DT>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) decode_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint32_t smem[];
    uint32_t *lut = smem;                       // [ctx][slot]
    uint32_t *cum = smem + kLutEntries;         // [ctx][257]
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;

    // ---- tables: sentinel everywhere (token 255, f = 2^11: an identity step), then the
    // cumulative frequencies per context (warps take contexts round robin), then the slots of
    // every token
    for (uint32_t i = threadIdx.x; i < kLutEntries; i += blockDim.x) lut[i] = (255u << 24) | (kProbScale << 12) | (i & (kProbScale - 1));
    for (uint32_t c = warp; c < uint32_t(kContexts); c += nwarps) {  // small CTAs take several contexts
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
        uint32_t lo = cum[c * 257 + t], f = cum[c * 257 + t + 1] - lo;
        uint32_t fill = f < kProbScale ? f : kProbScale;
        for (uint32_t s = lane; s < fill; s += 32)
            if (lo + s < kProbScale) lut[c * kProbScale + lo + s] = (t << 24) | (fill << 12) | s;
    }
    __syncthreads();

    // ---- tiles of this CTA: a contiguous range, warps round robin
    uint32_t t_begin = uint32_t(uint64_t(blockIdx.x) * p.T / gridDim.x);
    uint32_t t_end = uint32_t(uint64_t(blockIdx.x + 1) * p.T / gridDim.x);
    const uint32_t m0 = split_of(p.splits, 0), m1 = split_of(p.splits, 1), m2 = split_of(p.splits, 2);
    for (uint32_t t = t_begin + warp; t < t_end; t += nwarps) {
        uint32_t beg = __ldg(p.dir + t), end = __ldg(p.dir + t + 1);
        if (end < beg + 8 || uint64_t(end) > p.tile_units) {
            if (lane == 0 && p.status) atomicOr(p.status, EP_DEC_BAD_TILE);
            continue;
        }
        const uint8_t *tp = p.tiles + size_t(beg) * 16;
        Lane s;
        s.x = __ldg(reinterpret_cast<const uint32_t *>(tp) + lane);
        s.pos = 0;
        s.err = 0;
        s.nwords = (end - beg) * 8u - 64u;
        s.words = reinterpret_cast<const uint16_t *>(tp + 128);
        asm("mov.u32 %0, %%lanemask_lt;" : "=r"(s.lt));
        uint32_t b0 = t * 32u * p.K;
        uint32_t b = b0 + lane;
        uint32_t row = b / p.cb, col = b - row * p.cb;
        for (uint32_t k = 0; k < p.K; ++k, b0 += 32u, b += 32u) {
            if (b0 >= p.nb) break;
            bool act = b < p.nb;
            float fr = act ? __ldg(p.rowf + row) : 0.0f;
            Packer<DT> pk;
            // coordinate 0 carries the coset c
            int32_t v = unzigzag(decode_value(s, act, lut, m0));
            int32_t c = v & 1;
            int32_t y = (v - c) >> 1;
            int32_t par = y & 1;
            pk.put(0, v, fr);
            const uint32_t *lb = lut + (1u + uint32_t(c)) * kProbScale;
            uint32_t mb = c ? m2 : m1;
#pragma unroll
            for (int i = 1; i < 7; ++i) {
                y = unzigzag(decode_value(s, act, lb, mb));
                par ^= y & 1;
                pk.put(i, 2 * y + c, fr);
            }
            // coordinate 7: E8 forces y7 = par (mod 2)
            uint32_t c7 = 3u + 2u * uint32_t(c) + uint32_t(par);
            int32_t t7 = unzigzag(decode_value(s, act, lut + c7 * kProbScale, split_of(p.splits, c7)));
            pk.put(7, 2 * (2 * t7 + par) + c, fr);
            if (act) pk.store(p.out, b);
            col += 32u;
            while (col >= p.cb) {
                col -= p.cb;
                ++row;
            }
        }
        if (s.x != kStateLow) s.err |= EP_DEC_BAD_END;
        if (s.pos > s.nwords || s.nwords - s.pos >= 8u) s.err |= EP_DEC_WORD_COUNT;
        if (s.err && p.status) atomicOr(p.status, s.err);
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
                                                 int(kSmemBytes));
            if (e != cudaSuccess) return e;
            g_cache.attr[device][DT] = true;
        }
        sms = g_cache.sms[device];
    }
    uint32_t warps = (p.T + uint32_t(sms) - 1) / uint32_t(sms);
    warps = warps < 1 ? 1 : (warps > uint32_t(kMaxWarps) ? uint32_t(kMaxWarps) : warps);
    uint32_t grid = (p.T + warps - 1) / warps;
    if (grid > uint32_t(sms)) grid = uint32_t(sms);
    decode_kernel<DT><<<grid, warps * 32, kSmemBytes, stream>>>(p);
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
