// Tile-ANS decode for sm_100a: ep_ans_prepare and ep_ans_decompress, the lossless scheme of
// "EntroPack README", Configuration (TileANSConfig) on the lattice stream's tile machinery.
//   * ep_ans_prepare turns the stream's 256 frequencies into a 4096-slot table (16 KB): a slot's
//     32-bit entry holds the symbol's frequency (12 bits), the symbol (8 bits) and the slot's
//     offset inside the symbol (12 bits);
//   * ep_ans_decompress: one CTA per SM stages the table and each warp's tiles in shared memory
//     with bulk copies completing on mbarriers (as the lattice decode does); lane l of a tile runs
//     the rANS coder of lane l over its own word region, 8 symbols per chunk, and merges the
//     decoded top bytes with the chunk's raw bytes (one 8- or 24-byte load from the raw plane) by
//     byte permutes into one 16-byte (16-bit types), two 16-byte (FP32) or one 8-byte (8-bit
//     types) store per lane.  A warp stores 32 consecutive chunks per step.
// The path is a scan over compressed bytes: bound by HBM bandwidth and the rANS chain's latency,
// with no dense contraction and so no tensor cores.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/eptile.h"
#include "device_util.cuh"
#include "tile_ans.h"

namespace ep {
namespace ta {
namespace {

constexpr int kMaxWarps = 32;
constexpr uint32_t kSlack = 64;  // bytes past a tile that a lane's read-ahead may touch (8 words + 1)
constexpr size_t kBarBytes = size_t(kMaxWarps) * 2 * 8 + 16;
constexpr size_t kFixedBytes = kTableBytes + kBarBytes;
constexpr size_t kSmemLimit = 232448;
static_assert(kFixedBytes % 16 == 0, "tile buffers must start 16-byte aligned");

struct Params {
    const uint32_t *dir;
    const uint8_t *tiles;
    const uint8_t *raw;
    const uint32_t *table;
    uint8_t *out;
    uint32_t *status;
    uint64_t tile_units;
    uint64_t n;       // elements
    uint64_t nc;      // chunks of 8
    uint32_t K, T;
    uint32_t tile_buf, nbuf;
};

// one symbol: x' = f (x >> 12) + (slot - cum); below 2^16 the state takes the next word of the
// lane's region (read ahead, predicated).  Returns the slot entry.
__device__ __forceinline__ uint32_t ans_step(uint32_t &x, uint32_t &wp, uint32_t &w, uint32_t lut) {
    // slot address lut + 4 (x mod 2^12) = lut + 4x - 2^14 (x >> 12), exact modulo 2^32
    uint32_t xs = x >> kProbBits, a, t;
    asm("mad.lo.u32 %0, %1, 4, %2;" : "=r"(t) : "r"(x), "r"(lut));
    asm("mad.lo.u32 %0, %1, -16384, %2;" : "=r"(a) : "r"(xs), "r"(t));
    const uint32_t e = lds32(a);
    uint32_t xn = (e >> 20) * xs + (e & (kProbScale - 1u));
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.lt.u32 p, %0, 65536;\n\t@p mad.lo.u32 %0, %0, 65536, %2;\n\t"
        "@p add.u32 %1, %1, 2;\n\t@p ld.shared.u16 %2, [%1];\n\t}"
        : "+r"(xn), "+r"(wp), "+r"(w));
    x = xn;
    return e;
}

// the 8 decoded symbols (bits 12..19 of the entries) as 8 bytes, element order
__device__ __forceinline__ void pack_symbols(const uint32_t (&e)[8], uint32_t &lo, uint32_t &hi) {
    uint32_t u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) u[j] = e[j] >> 12;
    lo = __byte_perm(__byte_perm(u[0], u[1], 0x0040), __byte_perm(u[2], u[3], 0x0040), 0x5410);
    hi = __byte_perm(__byte_perm(u[4], u[5], 0x0040), __byte_perm(u[6], u[7], 0x0040), 0x5410);
}

// element j of chunk c: its low bytes from the raw plane and its top byte s
template <int ESZ>
__device__ __forceinline__ void store_element(const Params &p, uint64_t i, uint32_t s) {
    uint8_t *o = p.out + i * ESZ;
#pragma unroll
    for (int b = 0; b < ESZ - 1; ++b) o[b] = __ldg(p.raw + i * (ESZ - 1) + b);
    o[ESZ - 1] = uint8_t(s);
}

// the raw bytes of whole chunk c (8 for 16-bit types, 24 for FP32; none for 8-bit types), loaded
// two chunks ahead of their use so that the load's latency hides behind the rANS chain
template <int ESZ>
struct RawChunk {
    uint2 r[ESZ == 1 ? 1 : ESZ - 1];
};

template <int ESZ>
__device__ __forceinline__ RawChunk<ESZ> load_raw(const Params &p, uint64_t c, bool whole) {
    RawChunk<ESZ> R{};
    if constexpr (ESZ > 1) {
        const uint2 *rp = reinterpret_cast<const uint2 *>(p.raw + (ESZ - 1) * 8 * c);
#pragma unroll
        for (int q = 0; q < ESZ - 1; ++q) R.r[q] = whole ? __ldg(rp + q) : make_uint2(0u, 0u);
    }
    return R;
}

// chunk c: merge and store (whole chunks as vectors; the tensor's last, partial chunk element by
// element)
template <int ESZ>
__device__ __forceinline__ void store_chunk(const Params &p, uint64_t c, const uint32_t (&e)[8], const RawChunk<ESZ> &R) {
    uint32_t lo, hi;
    pack_symbols(e, lo, hi);
    if (8 * c + 8 > p.n) {
        const uint32_t k = uint32_t(p.n - 8 * c);
#pragma unroll
        for (uint32_t j = 0; j < 8; ++j)  // constant indices keep e[] in registers
            if (j < k) store_element<ESZ>(p, 8 * c + j, (e[j] >> 12) & 0xffu);
        return;
    }
    if constexpr (ESZ == 1) {
        reinterpret_cast<uint2 *>(p.out)[c] = make_uint2(lo, hi);
    } else if constexpr (ESZ == 2) {
        // bytes r0..r7 of the raw plane, then [r0 s0 r1 s1] [r2 s2 r3 s3] ...
        const uint2 r = R.r[0];
        reinterpret_cast<uint4 *>(p.out)[c] =
            make_uint4(__byte_perm(r.x, lo, 0x5140), __byte_perm(r.x, lo, 0x7362), __byte_perm(r.y, hi, 0x5140),
                       __byte_perm(r.y, hi, 0x7362));
    } else {
        // 24 raw bytes: element j's low three bytes start at byte 3j
        const uint32_t W[7] = {R.r[0].x, R.r[0].y, R.r[1].x, R.r[1].y, R.r[2].x, R.r[2].y, 0u};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t low = __funnelshift_r(W[(3 * j) / 4], W[(3 * j) / 4 + 1], 8 * ((3 * j) % 4)) & 0xffffffu;
            o[j] = low | (e[j] >> 12) << 24;
        }
        uint4 *op = reinterpret_cast<uint4 *>(p.out) + 2 * c;
        op[0] = make_uint4(o[0], o[1], o[2], o[3]);
        op[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// Decodes tile t with one warp from the warp's shared-memory buffer at `head`.  Returns EP_DEC_*
// bits of this lane.
template <int ESZ>
__device__ __forceinline__ uint32_t decode_tile(const Params &p, uint32_t lut, uint32_t head, uint32_t tile_bytes,
                                                uint32_t t, uint32_t lane) {
    uint32_t x = lds32(head + 4u * lane);
    const uint32_t len = lds16(head + 128u + 2u * lane);
    uint32_t incl = len;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= uint32_t(d)) incl += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    const uint32_t capacity = (tile_bytes - uint32_t(kTileHead)) / 2u;
    if (total > capacity) return EP_DEC_WORD_OVERRUN;  // warp-uniform: the regions overrun the tile
    const uint32_t start = incl - len;
    const uint32_t area = head + uint32_t(kTileHead);
    uint32_t wp = area + 2u * start, w = lds16(wp);
    const uint32_t wlim = area + 2u * capacity;
    uint32_t err = 0;
    uint64_t c = uint64_t(t) * 32u * p.K + lane;
    // the raw bytes of the lane's chunk at step k + j, j = 0, 1 (zero past the lane's chunks)
    auto raw_at = [&](uint32_t k, uint64_t ck) {
        return k < p.K && ck < p.nc ? load_raw<ESZ>(p, ck, 8 * ck + 8 <= p.n) : RawChunk<ESZ>{};
    };
    RawChunk<ESZ> R0 = raw_at(0, c), R1 = raw_at(1, c + 32u);
    for (uint32_t k = 0; k < p.K; ++k, c += 32u) {
        const bool act = c < p.nc;
        if (!__any_sync(0xffffffffu, act)) break;
        // a damaged stream may drive a lane's reads ahead (at most one word per symbol): stop
        // before they leave the buffer's slack
        if (__any_sync(0xffffffffu, wp > wlim)) {
            err |= EP_DEC_WORD_OVERRUN;
            break;
        }
        const RawChunk<ESZ> R2 = raw_at(k + 2, c + 64u);
        if (act) {
            uint32_t e[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) e[j] = ans_step(x, wp, w, lut);
            store_chunk<ESZ>(p, c, e, R0);
        }
        R0 = R1;
        R1 = R2;
    }
    if (err) return err;
    if (x != kStateLow) err |= EP_DEC_BAD_END;
    const uint32_t used = (wp - area) / 2u - start;
    if (used != len) err |= used > len ? EP_DEC_WORD_OVERRUN : EP_DEC_WORD_COUNT;
    if (capacity - total >= 8u) err |= EP_DEC_WORD_COUNT;
    return err;
}

template <int ESZ>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) ans_decode_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const uint32_t lut = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const uint32_t bars = lut + uint32_t(kTableBytes);
    const uint32_t tbar = bars + uint32_t(kMaxWarps) * 16u;
    const uint32_t nbuf = p.nbuf;
    const uint32_t bufs = bars + uint32_t(kBarBytes) + warp * nbuf * p.tile_buf;
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
    // launched with programmatic stream serialisation: nothing global is touched before the
    // previous kernel's writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        mbar_expect(tbar, uint32_t(kTableBytes));
        bulk_g2s(lut, p.table, uint32_t(kTableBytes), tbar);
    }
    __syncthreads();
    auto tile_ok = [&](uint32_t t, uint32_t &beg, uint32_t &bytes) -> bool {
        beg = __ldg(p.dir + t);
        const uint32_t end = __ldg(p.dir + t + 1);
        bytes = (end - beg) * 16u;
        return end >= beg + uint32_t(kTileHead / 16) && uint64_t(end) <= p.tile_units &&
               bytes + kSlack <= p.tile_buf;
    };
    auto issue = [&](uint32_t t, uint32_t j) -> bool {
        uint32_t beg, bytes;
        const bool ok = tile_ok(t, beg, bytes);
        if (ok && lane == 0) {
            const uint32_t bar = bars + 16u * warp + 8u * j;
            fence_proxy_async();
            mbar_expect(bar, bytes);
            bulk_g2s(bufs + j * p.tile_buf, p.tiles + size_t(beg) * 16, bytes, bar);
        }
        return ok;
    };
    uint32_t pend = 0, phase = 0;
    for (uint32_t j = 0; j < nbuf; ++j) {
        const uint32_t t = t_begin + warp + j * nwarps;
        if (t < t_end && issue(t, j)) pend |= 1u << j;
    }
    const bool tables_ok = mbar_wait(tbar, 0);
    if (!tables_ok && lane == 0 && p.status) atomicOr(p.status, EP_DEC_TIMEOUT);
    uint32_t j = 0;
    for (uint32_t t = t_begin + warp; t < t_end; t += nwarps, ++j) {
        const uint32_t b = j % nbuf;
        uint32_t beg, bytes, err = 0;
        if (!tile_ok(t, beg, bytes)) {
            err = EP_DEC_BAD_TILE;
        } else if (pend & (1u << b)) {
            const bool done = mbar_wait(bars + 16u * warp + 8u * b, (phase >> b) & 1u);
            phase ^= 1u << b;
            pend &= ~(1u << b);
            if (!done) {  // a lost copy: report, let the other buffer's copy land, stop
                if (lane == 0 && p.status) atomicOr(p.status, EP_DEC_TIMEOUT);
                const uint32_t o = b ^ 1u;
                if (nbuf > 1 && (pend & (1u << o))) mbar_wait(bars + 16u * warp + 8u * o, (phase >> o) & 1u);
                return;
            }
            if (tables_ok) err = decode_tile<ESZ>(p, lut, bufs + b * p.tile_buf, bytes, t, lane);
        } else {
            err = EP_DEC_BAD_TILE;
        }
        if (err && p.status) atomicOr(p.status, err);
        __syncwarp();
        const uint32_t tn = t + nbuf * nwarps;
        if (tn < t_end && issue(tn, b)) pend |= 1u << b;
    }
}

// the slot table: one CTA per 256 slots; the 256 frequencies' prefix sums in shared memory, then
// each thread finds its slot's symbol by binary search
__global__ void __launch_bounds__(256) ans_prepare_kernel(const uint16_t *freq, uint32_t *table, uint32_t *status) {
    __shared__ uint32_t cum[257];
    __shared__ uint32_t part[8];
    const uint32_t i = threadIdx.x, lane = i & 31u, warp = i >> 5;
    const uint32_t f0 = freq[i];
    const uint32_t f = min(f0, kProbScale);
    uint32_t incl = f;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= uint32_t(d)) incl += y;
    }
    if (lane == 31) part[warp] = incl;
    __syncthreads();
    uint32_t before = 0, all = 0;
    for (uint32_t w = 0; w < 8; ++w) {
        before += w < warp ? part[w] : 0u;
        all += part[w];
    }
    cum[i] = before + incl - f;
    if (i == 0) cum[256] = all;
    __syncthreads();
    const bool bad = __syncthreads_or(f0 >= kProbScale || all != kProbScale);
    if (bad && i == 0 && blockIdx.x == 0 && status) atomicOr(status, EP_DEC_BAD_TOKEN);
    const uint32_t slot = blockIdx.x * 256u + i;
    uint32_t lo = 0, hi = 256;  // the last symbol s with cum[s] <= slot (symbols with f = 0 skipped)
    while (hi - lo > 1) {
        const uint32_t mid = (lo + hi) >> 1;
        if (cum[mid] <= slot)
            lo = mid;
        else
            hi = mid;
    }
    const uint32_t fs = min(cum[lo + 1] - cum[lo], kProbScale - 1u);
    table[slot] = (fs << 20) | (lo << 12) | ((slot - cum[lo]) & (kProbScale - 1u));
}

struct DeviceCache {
    std::mutex mu;
    int sms[64] = {0};
    bool attr[64][5] = {};
};
DeviceCache g_cache;

template <int ESZ>
cudaError_t launch(Params &p, uint64_t max_tile, int device, cudaStream_t stream) {
    int sms;
    {
        std::lock_guard<std::mutex> g(g_cache.mu);
        if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
        if (!g_cache.sms[device]) {
            const cudaError_t e = cudaDeviceGetAttribute(&g_cache.sms[device], cudaDevAttrMultiProcessorCount, device);
            if (e != cudaSuccess) return e;
        }
        if (!g_cache.attr[device][ESZ]) {
            const cudaError_t e =
                cudaFuncSetAttribute(ans_decode_kernel<ESZ>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemLimit));
            if (e != cudaSuccess) return e;
            g_cache.attr[device][ESZ] = true;
        }
        sms = g_cache.sms[device];
    }
    // one CTA per SM (at most one per tile), warps = tiles per CTA within kMaxWarps; two staging
    // buffers per warp when a warp has several tiles and they fit, else one; fewer warps when even
    // one buffer per warp does not fit
    const uint32_t grid = p.T < uint32_t(sms) ? p.T : uint32_t(sms);
    uint32_t warps = (p.T + grid - 1) / grid;
    warps = warps > uint32_t(kMaxWarps) ? uint32_t(kMaxWarps) : warps;
    const size_t avail = kSmemLimit - kFixedBytes;
    p.tile_buf = uint32_t((max_tile + kSlack + 15) & ~uint64_t(15));
    if (p.tile_buf > avail) return cudaErrorInvalidValue;  // the caller reports EP_ERR_UNSUPPORTED
    const bool many = p.T > grid * warps;
    if (many && 2ull * warps * p.tile_buf <= avail) {
        p.nbuf = 2;
    } else {
        p.nbuf = 1;
        if (uint64_t(warps) * p.tile_buf > avail) warps = uint32_t(avail / p.tile_buf);
    }
    if (warps < 1) warps = 1;
    const size_t smem = kFixedBytes + size_t(warps) * p.nbuf * p.tile_buf;
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
    return cudaLaunchKernelEx(&cfg, ans_decode_kernel<ESZ>, p);
}

int check_info(const ep_ans_info *info) {
    if (info->n_elems <= 0 || info->n_tiles == 0 || info->blocks_per_lane == 0) return EP_ERR_INVALID_ARG;
    if (elt_bytes(info->dtype) == 0) return EP_ERR_CORRUPT;
    if (info->workspace_nbytes < kTableBytes) return EP_ERR_INVALID_ARG;
    return EP_OK;
}

}  // namespace
}  // namespace ta
}  // namespace ep

extern "C" int ep_ans_prepare(const ep_ans_info *info, const void *d_blob, void *d_workspace, uint32_t *d_status,
                              ep_stream_t stream) {
    using namespace ep::ta;
    if (!info || !d_blob || !d_workspace) return EP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_blob) | reinterpret_cast<uintptr_t>(d_workspace)) & 15u) return EP_ERR_INVALID_ARG;
    const int rc = check_info(info);
    if (rc != EP_OK) return rc;
    const uint16_t *freq = reinterpret_cast<const uint16_t *>(static_cast<const uint8_t *>(d_blob) + info->off_freq);
    ans_prepare_kernel<<<kProbScale / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        freq, static_cast<uint32_t *>(d_workspace), d_status);
    return cudaGetLastError() == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

extern "C" int ep_ans_decompress(const ep_ans_info *info, const void *d_blob, const void *d_workspace, void *d_out,
                                 uint32_t *d_status, ep_stream_t stream) {
    using namespace ep::ta;
    if (!info || !d_blob || !d_workspace || !d_out) return EP_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d_blob) | reinterpret_cast<uintptr_t>(d_out) |
         reinterpret_cast<uintptr_t>(d_workspace)) & 15u)
        return EP_ERR_INVALID_ARG;
    const int rc = check_info(info);
    if (rc != EP_OK) return rc;
    const uint8_t *base = static_cast<const uint8_t *>(d_blob);
    Params p;
    p.dir = reinterpret_cast<const uint32_t *>(base + info->off_dir);
    p.tiles = base + info->off_tiles;
    p.raw = base + info->off_raw;
    p.table = static_cast<const uint32_t *>(d_workspace);
    p.out = static_cast<uint8_t *>(d_out);
    p.status = d_status;
    p.tile_units = (info->storage_nbytes - info->off_tiles) / 16;
    p.n = uint64_t(info->n_elems);
    p.nc = (p.n + kChunk - 1) / kChunk;
    p.K = info->blocks_per_lane;
    p.T = info->n_tiles;
    int device;
    if (cudaGetDevice(&device) != cudaSuccess) return EP_ERR_CUDA;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch (elt_bytes(info->dtype)) {
    case 1: e = launch<1>(p, info->max_tile_nbytes, device, s); break;
    case 2: e = launch<2>(p, info->max_tile_nbytes, device, s); break;
    case 4: e = launch<4>(p, info->max_tile_nbytes, device, s); break;
    default: return EP_ERR_CORRUPT;
    }
    if (e == cudaErrorInvalidValue) return EP_ERR_UNSUPPORTED;
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
