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
#include <mutex>

#include "decode_core.cuh"

namespace ep {
namespace {

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
