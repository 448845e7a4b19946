// Device compressor: ep_compress_device.
//
// compress(tensor, config) of the "EntroPack API reference" with the tensor already in device
// memory.  The pipeline is the host compressor's (the "EntroPack" Abstract: row-normalized E8
// lattice quantization, a conditional model of the coordinates, a resolution picked by sampled
// storage estimates, tiles of interleaved rANS), with the work over elements, blocks and lanes on
// the GPU:
//   * rows_kernel      one lane per row over 32x32 shared-memory tiles: finite check, INT8 / FP8
//                      codes and scales, the row RMS summed left to right in double (the order is
//                      part of the result);
//   * quant_kernel     per block: x = w / (2 f_r), E8 nearest point, symbols and contexts, and a
//                      histogram of the values' bit lengths per context;
//   * token_kernel     per coordinate: its token at the chosen splits, token counts per context
//                      and the raw extra bits;
//   * pair_kernel      per block of a paired stream: counts of the token pairs of coordinates
//                      (1,2), (3,4), (5,6);
//   * lane_kernel      one thread per (tile, lane), twice: the lane's rANS encode (tokens in
//                      reverse) and raw bits, first counting words, then writing them in decode
//                      order into the lane's region of the tile.
// The decisions in between (splits, frequency tables, the estimate, the bisection over the
// resolution, tile offsets) are taken on the host by the same functions the host compressor
// uses, from integer histograms, so the stream equals the host compressor's byte for byte.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "../../include/eptile.h"
#include "encode_host.h"
#include "encode_math.h"
#include "format.h"

namespace ep {
namespace {

constexpr int kLenBins = 33;  // bit lengths 0..32
// frequency tables as the lane kernel holds them: one row per context, long enough for a pair table
constexpr uint32_t kTableStride = kPairMaxTable > kMaxAlphabet ? kPairMaxTable : kMaxAlphabet;
constexpr uint32_t kPairBins = kPairBaseMax * kPairBaseMax;

struct DevSrc {
    const void *p;
    int dt;
};

__device__ __forceinline__ float src_at(const DevSrc &s, int64_t i) {
    if (s.dt == EP_BF16) return __uint_as_float(uint32_t(static_cast<const uint16_t *>(s.p)[i]) << 16);
    if (s.dt == EP_FP16) return __half2float(static_cast<const __half *>(s.p)[i]);
    return static_cast<const float *>(s.p)[i];
}

// the value the quantizer sees: the code (INT8 / FP8 containers) or the source element
__device__ __forceinline__ double value_at(const DevSrc &s, const float *codes, int64_t i) {
    return codes ? double(codes[i]) : double(src_at(s, i));
}

__device__ __forceinline__ uint32_t low_of(uint32_t c) { return c == 0 ? 2u : (c < 3 ? 1u : 0u); }

struct Splits {
    uint32_t m[kContexts];
};

// ------------------------------------------------------------------ rows
// A warp owns 32 rows, lane l row row0 + l.  Columns go through shared memory 32 at a time: the
// warp loads a 32x32 tile row by row (coalesced), then every lane walks its own row's 32 values in
// column order, so the RMS is still summed left to right in double.  Tile rows are padded to 33
// words (conflict-free column walks).
constexpr int kRowWarps = 8;

__global__ void __launch_bounds__(kRowWarps * 32) rows_kernel(DevSrc src, int64_t rows, int64_t cols,
                                                                int container, float *codes, float *scales,
                                                                float *rms, uint32_t *bad) {
    __shared__ float tile[kRowWarps][32][33];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t row0 = (int64_t(blockIdx.x) * kRowWarps + wid) * 32;
    if (row0 >= rows) return;  // the whole warp
    float(*t)[33] = tile[wid];
    const int64_t r = row0 + lane;
    const bool live = r < rows;
    const int nr = int(rows - row0 < 32 ? rows - row0 : 32);
    auto load = [&](int64_t c0, int nc) {  // t[rr][j] = source element (row0 + rr, c0 + j)
        for (int rr = 0; rr < nr; ++rr)
            if (lane < nc) t[rr][lane] = src_at(src, (row0 + rr) * cols + c0 + lane);
        __syncwarp();
    };
    bool nonfinite = false;
    double amax = 0.0, acc = 0.0;
    float s = 1.0f;
    if (codes) {
        // per-row absmax codes: symmetric INT8 [-127, 127] or E4M3 with saturation at 448
        for (int64_t c0 = 0; c0 < cols; c0 += 32) {
            const int nc = int(cols - c0 < 32 ? cols - c0 : 32);
            load(c0, nc);
            if (live)
                for (int j = 0; j < nc; ++j) {
                    const float w = t[lane][j];
                    nonfinite |= !isfinite(w);
                    amax = fmax(amax, fabs(double(w)));
                }
            __syncwarp();
        }
        const double bound = container == EP_INT8 ? 127.0 : 448.0;
        s = amax > 0.0 ? float(ddiv(amax, bound)) : 1.0f;
        if (s == 0.0f) s = FLT_MIN;
        if (live) scales[r] = s;
    }
    for (int64_t c0 = 0; c0 < cols; c0 += 32) {
        const int nc = int(cols - c0 < 32 ? cols - c0 : 32);
        load(c0, nc);
        if (live)
            for (int j = 0; j < nc; ++j) {
                double a = t[lane][j];
                if (codes) {
                    if (amax == 0.0)
                        a = 0.0;
                    else if (container == EP_INT8)
                        a = fmin(127.0, fmax(-127.0, dround(ddiv(a, double(s)))));
                    else
                        a = e4m3_round(float(ddiv(a, double(s))));
                    t[lane][j] = float(a);
                } else {
                    nonfinite |= !isfinite(float(a));
                }
                acc = dadd(acc, dmul(a, a));
            }
        __syncwarp();
        if (codes)  // write the tile's codes back, row by row (coalesced)
            for (int rr = 0; rr < nr; ++rr)
                if (lane < nc) codes[(row0 + rr) * cols + c0 + lane] = t[rr][lane];
        __syncwarp();
    }
    if (live) rms[r] = float(__dsqrt_rn(ddiv(acc, double(cols))));
    if (nonfinite) atomicOr(bad, 1u);
}

// ------------------------------------------------------------------ blocks
// items j = 0..n-1 are blocks j * step (every block, or the estimate's sample); rows are
// zero-padded to whole blocks
__global__ void quant_kernel(DevSrc src, const float *codes, int64_t cols, int64_t cb, const float *rms, int k,
                             int64_t step, int64_t n, uint8_t *ctx, uint32_t *val, unsigned long long *by_len) {
    __shared__ unsigned int h[kContexts * kLenBins];
    for (int i = threadIdx.x; i < kContexts * kLenBins; i += blockDim.x) h[i] = 0;
    __syncthreads();
    for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j < n; j += int64_t(gridDim.x) * blockDim.x) {
        const int64_t b = j * step, r = b / cb, c0 = 8 * (b - r * cb), base = r * cols + c0;
        const int n8 = int(cols - c0 < 8 ? cols - c0 : 8);
        const float f = factor_of(rms[r], k);
        int32_t v[8];
        if (f == 0.0f) {
            for (int i = 0; i < 8; ++i) v[i] = 0;
        } else {
            double x[8];
            const double two_f = dmul(2.0, double(f));
            for (int i = 0; i < 8; ++i) x[i] = i < n8 ? ddiv(value_at(src, codes, base + i), two_f) : 0.0;
            quantize_e8(x, v);
        }
        uint8_t cx[8];
        uint32_t s[8];
        symbols_of(v, cx, s);
        for (int i = 0; i < 8; ++i) {
            ctx[8 * j + i] = cx[i];
            val[8 * j + i] = s[i];
            atomicAdd(&h[cx[i] * kLenBins + bitlen(s[i])], 1u);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kContexts * kLenBins; i += blockDim.x)
        if (h[i]) atomicAdd(&by_len[i], (unsigned long long)h[i]);
}

// token counts per context (kMaxAlphabet bins each) and the raw extra bits of items 0..n-1
__global__ void token_kernel(const uint8_t *ctx, const uint32_t *val, int64_t n, Splits sp, unsigned long long *cnt,
                             unsigned long long *extra) {
    __shared__ unsigned int h[kContexts * kMaxAlphabet];
    for (int i = threadIdx.x; i < kContexts * int(kMaxAlphabet); i += blockDim.x) h[i] = 0;
    __syncthreads();
    unsigned long long bits = 0;
    for (int64_t s = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; s < 8 * n; s += int64_t(gridDim.x) * blockDim.x) {
        const uint32_t c = ctx[s];
        const Token t = token_of(val[s], sp.m[c], low_of(c));
        atomicAdd(&h[c * kMaxAlphabet + t.tok], 1u);
        bits += t.nbits;
    }
    for (int d = 16; d > 0; d >>= 1) bits += __shfl_down_sync(0xffffffffu, bits, d);
    if ((threadIdx.x & 31) == 0 && bits) atomicAdd(extra, bits);
    __syncthreads();
    for (int i = threadIdx.x; i < kContexts * int(kMaxAlphabet); i += blockDim.x)
        if (h[i]) atomicAdd(&cnt[i], (unsigned long long)h[i]);
}

// counts of the token pairs inside the bases of contexts 1 and 2 (B1 x B1 and B2 x B2 bins at
// offsets 0 and kPairBins)
__global__ void pair_kernel(const uint8_t *ctx, const uint32_t *val, int64_t nb, Splits sp, uint32_t B1, uint32_t B2,
                            unsigned long long *pc) {
    __shared__ unsigned int h[2 * kPairBins];
    for (int i = threadIdx.x; i < int(2 * kPairBins); i += blockDim.x) h[i] = 0;
    __syncthreads();
    for (int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; b < nb; b += int64_t(gridDim.x) * blockDim.x) {
        const uint32_t c = ctx[8 * b + 1];  // 1 or 2
        const uint32_t B = c == 1 ? B1 : B2;
        for (int j = 0; j < 3; ++j) {
            const uint32_t ta = token_of(val[8 * b + 1 + 2 * j], sp.m[c], 1).tok;
            const uint32_t tb = token_of(val[8 * b + 2 + 2 * j], sp.m[c], 1).tok;
            if (ta < B && tb < B) atomicAdd(&h[(c - 1) * kPairBins + ta * B + tb], 1u);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < int(2 * kPairBins); i += blockDim.x)
        if (h[i]) atomicAdd(&pc[i], (unsigned long long)h[i]);
}

// ------------------------------------------------------------------ lanes
// One thread per (tile, lane); a warp is a tile.  Lane l of tile t codes blocks t 32 K + 32 k + l.
// Its region holds the rANS words in decode order, then its raw extra bits packed least
// significant bit first into 16-bit words stored back to front.  WRITE = false: count the words
// and keep the final state; WRITE = true: write state, count and words into the tile.
struct LaneArgs {
    const uint8_t *ctx;
    const uint32_t *val;
    const uint16_t *freq;   // kContexts x kTableStride (paired contexts 1, 2: the pair tables)
    const uint16_t *cum;    // kContexts x kTableStride
    uint32_t *count;        // T x 32: words of each lane's region
    uint32_t *rwords;       // T x 32: of which rANS words
    uint32_t *state;        // T x 32: final encoder state (the decoder's initial state)
    uint32_t *too_long;     // set when a region exceeds 65535 words
    const uint32_t *dir;    // T + 1 tile offsets in 16-byte units (WRITE)
    uint8_t *tiles;         // tile section of the output (WRITE)
    int64_t nb;
    uint32_t K, T;
    int64_t cb;             // blocks per row
    int layout;             // block order of the tiles (format.h lane_block)
    Splits sp;
    uint32_t paired;
    uint32_t B[kContexts];     // paired contexts 1, 2: pair base min(A, 40)
    uint32_t rawb[kContexts];  // paired contexts 1, 2: raw bits of one token of an escaped pair
};

// A block's rANS symbols in decode order (context row, symbol, table bits) and, through `push`,
// its raw bits: single coding, the 8 tokens; paired coding, token 0, the three pair symbols
// (a pair with a token outside the base B, or whose table entry is 0, is the escape B * B) and
// token 7, the escaped pairs' tokens leading the raw bits.  Returns the symbol count.
struct Sym {
    uint32_t c, s, bits;
};
template <typename Push>
__device__ __forceinline__ int block_syms(const LaneArgs &a, const uint16_t *sf, int64_t b, Sym *sym, Push push) {
    Token tk[8];
    uint32_t cx[8];
    for (int i = 0; i < 8; ++i) {
        cx[i] = a.ctx[8 * b + i];
        tk[i] = token_of(a.val[8 * b + i], a.sp.m[cx[i]], low_of(cx[i]));
    }
    int n = 0;
    if (!a.paired) {
        for (int i = 0; i < 8; ++i) sym[n++] = {cx[i], tk[i].tok, kProbBits};
    } else {
        const uint32_t pc = cx[1], B = a.B[pc];
        bool esc[3];
        sym[n++] = {cx[0], tk[0].tok, kProbBits};
        for (int j = 0; j < 3; ++j) {
            const uint32_t ta = tk[1 + 2 * j].tok, tb = tk[2 + 2 * j].tok;
            esc[j] = ta >= B || tb >= B || sf[pc * kTableStride + ta * B + tb] == 0;
            sym[n++] = {pc, esc[j] ? B * B : ta * B + tb, kPairBits};
        }
        sym[n++] = {cx[7], tk[7].tok, kProbBits};
        for (int j = 0; j < 3; ++j)
            if (esc[j]) {
                push(tk[1 + 2 * j].tok, a.rawb[pc]);
                push(tk[2 + 2 * j].tok, a.rawb[pc]);
            }
    }
    for (int i = 0; i < 8; ++i) push(tk[i].extra, tk[i].nbits);
    return n;
}

template <bool WRITE>
__global__ void lane_kernel(LaneArgs a) {
    __shared__ uint16_t sf[kContexts * kTableStride], sc[kContexts * kTableStride];
    for (int i = threadIdx.x; i < kContexts * int(kTableStride); i += blockDim.x) {
        sf[i] = a.freq[i];
        sc[i] = a.cum[i];
    }
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31u;
    const uint64_t t = (uint64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (t >= a.T) return;  // whole warps leave together
    // blocks of this lane, in the layout's order
    auto blk = [&](uint32_t k) { return lane_block(a.layout, a.cb, int64_t(t), int(lane), a.K, k); };
    uint32_t nk = 0;
    while (nk < a.K && blk(nk) < a.nb) ++nk;

    uint32_t n = 0, nr = 0, start = 0;
    uint16_t *area = nullptr;
    if (WRITE) {
        n = a.count[t * 32 + lane];
        nr = a.rwords[t * 32 + lane];
        uint32_t incl = n;
        for (int d = 1; d < 32; d <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= uint32_t(d)) incl += y;
        }
        start = incl - n;
        uint8_t *tile = a.tiles + size_t(a.dir[t]) * 16;
        const uint32_t x0 = a.state[t * 32 + lane];
        for (int b = 0; b < 4; ++b) tile[4 * lane + b] = uint8_t(x0 >> (8 * b));
        tile[4 * 32 + 2 * lane] = uint8_t(n);
        tile[4 * 32 + 2 * lane + 1] = uint8_t(n >> 8);
        area = reinterpret_cast<uint16_t *>(tile + kTileHead);
    }
    // raw bits, forward
    uint64_t acc = 0;
    uint32_t nacc = 0, raw = 0;
    auto push = [&](uint32_t v, uint32_t nbits) {
        acc |= uint64_t(v) << nacc;
        nacc += nbits;
        while (nacc >= 16) {
            if (WRITE) area[start + n - 1 - raw] = uint16_t(acc);
            ++raw;
            acc >>= 16;
            nacc -= 16;
        }
    };
    auto skip = [](uint32_t, uint32_t) {};
    Sym sym[8];
    for (uint32_t k = 0; k < nk; ++k) block_syms(a, sf, blk(k), sym, push);
    if (nacc) {
        if (WRITE) area[start + n - 1 - raw] = uint16_t(acc);
        ++raw;
    }
    // rANS, symbols in reverse; the i-th word emitted is word nr - 1 - i in decode order
    uint32_t x = kStateLow, emitted = 0;
    for (uint32_t k = nk; k-- > 0;) {
        const int ns = block_syms(a, sf, blk(k), sym, skip);
        for (int i = ns - 1; i >= 0; --i) {
            const uint32_t at = sym[i].c * kTableStride + sym[i].s, nbits = sym[i].bits;
            const uint32_t f = sf[at], cu = sc[at];
            if (uint64_t(x) >= (uint64_t(f) << (32 - nbits))) {  // keep the next state below 2^32
                if (WRITE) area[start + nr - 1 - emitted] = uint16_t(x);
                ++emitted;
                x >>= 16;
            }
            x = (x / f) * (1u << nbits) + (x % f) + cu;
        }
    }
    if (!WRITE) {
        a.count[t * 32 + lane] = emitted + raw;
        a.rwords[t * 32 + lane] = emitted;
        a.state[t * 32 + lane] = x;
        if (emitted + raw > 0xffffu) atomicOr(a.too_long, 1u);
    }
}

}  // namespace
}  // namespace ep

// ------------------------------------------------------------------ host side
namespace ep {
namespace {

size_t al256(size_t n) { return (n + 255) & ~size_t(255); }

// caller scratch, carved in this order (each piece 256-byte aligned)
struct Scratch {
    float *codes, *scales, *rms;
    uint8_t *ctx;
    uint32_t *val;
    unsigned long long *by_len, *cnt, *extra, *pairs;
    uint32_t *bad, *too_long;
    uint16_t *freq, *cum;
    uint32_t *count, *rwords, *state, *dir;
    size_t bytes;
};

Scratch carve(uint8_t *base, int64_t rows, int64_t cols, int container, int64_t nb, uint32_t T) {
    Scratch S{};
    size_t at = 0;
    auto take = [&](size_t n) {
        uint8_t *p = base ? base + at : nullptr;
        at += al256(n);
        return p;
    };
    S.codes = reinterpret_cast<float *>(take(is_code_container(container) ? size_t(rows * cols) * 4 : 0));
    S.scales = reinterpret_cast<float *>(take(size_t(rows) * 4));
    S.rms = reinterpret_cast<float *>(take(size_t(rows) * 4));
    S.ctx = take(size_t(nb) * 8);
    S.val = reinterpret_cast<uint32_t *>(take(size_t(nb) * 32));
    S.by_len = reinterpret_cast<unsigned long long *>(take(kContexts * kLenBins * 8));
    S.cnt = reinterpret_cast<unsigned long long *>(take(kContexts * kMaxAlphabet * 8));
    S.extra = reinterpret_cast<unsigned long long *>(take(8));
    S.pairs = reinterpret_cast<unsigned long long *>(take(2 * kPairBins * 8));
    S.bad = reinterpret_cast<uint32_t *>(take(4));
    S.too_long = reinterpret_cast<uint32_t *>(take(4));
    S.freq = reinterpret_cast<uint16_t *>(take(kContexts * kTableStride * 2));
    S.cum = reinterpret_cast<uint16_t *>(take(kContexts * kTableStride * 2));
    S.count = reinterpret_cast<uint32_t *>(take(size_t(T) * 32 * 4));
    S.rwords = reinterpret_cast<uint32_t *>(take(size_t(T) * 32 * 4));
    S.state = reinterpret_cast<uint32_t *>(take(size_t(T) * 32 * 4));
    S.dir = reinterpret_cast<uint32_t *>(take(size_t(T + 1) * 4));
    if (!is_code_container(container)) S.codes = nullptr;
    S.bytes = at;
    return S;
}

struct Plan {
    int64_t rows, cols, cb, nb;
    int src_dt, container, coding, layout;
    uint32_t K, T;
    bool ok;
};

Plan plan_of(int64_t rows, int64_t cols, int32_t src_dtype, const ep_config *cfg) {
    Plan P{};
    P.rows = rows;
    P.cols = cols;
    P.cb = (cols + 7) / 8;
    P.nb = rows * P.cb;
    P.src_dt = src_dtype;
    P.container = cfg->container_dtype ? cfg->container_dtype : src_dtype;
    P.coding = cfg->coding;
    P.layout = cfg->layout;
    P.K = cfg->blocks_per_lane ? cfg->blocks_per_lane
                               : (P.layout == kLayoutGemm ? 32u : auto_blocks_per_lane(P.nb, cfg->target_bpp));
    P.T = P.K ? uint32_t((P.nb + 32 * int64_t(P.K) - 1) / (32 * int64_t(P.K))) : 0;
    P.ok = P.K > 0 && (P.layout == kLayoutRows || P.layout == kLayoutGemm) && layout_fits(P.layout, rows, cols, P.K);
    return P;
}

struct Run {
    const Plan &P;
    DevSrc src;
    Scratch S;
    cudaStream_t st;
    int grid;
    cudaError_t err = cudaSuccess;

    void check(cudaError_t e) {
        if (err == cudaSuccess) err = e;
    }
    template <typename T>
    void d2h(T *h, const T *d, size_t n) {
        check(cudaMemcpyAsync(h, d, n * sizeof(T), cudaMemcpyDeviceToHost, st));
        check(cudaStreamSynchronize(st));
    }
    template <typename T>
    void h2d(T *d, const T *h, size_t n) {
        check(cudaMemcpyAsync(d, h, n * sizeof(T), cudaMemcpyHostToDevice, st));
    }
    int blocks_for(int64_t n, int per) const {
        int64_t b = (n + per - 1) / per;
        return int(b < 1 ? 1 : (b > grid ? grid : b));
    }

    // quantize items (every `step`-th block) at resolution k; returns the splits picked on them
    Splits quantize(int k, int64_t step, int64_t n) {
        check(cudaMemsetAsync(S.by_len, 0, kContexts * kLenBins * 8, st));
        quant_kernel<<<blocks_for(n, 256), 256, 0, st>>>(src, S.codes, P.cols, P.cb, S.rms, k, step, n, S.ctx, S.val,
                                                         S.by_len);
        check(cudaGetLastError());
        std::vector<unsigned long long> h(kContexts * kLenBins);
        d2h(h.data(), S.by_len, h.size());
        Splits sp;
        for (int c = 0; c < kContexts; ++c) {
            uint64_t by_len[kLenBins];
            for (int i = 0; i < kLenBins; ++i) by_len[i] = h[size_t(c * kLenBins + i)];
            sp.m[c] = pick_split(by_len, c);
        }
        return sp;
    }

    // token counts of items 0..n-1 at the splits, one vector per context (the alphabet's length)
    uint64_t tokens(const Splits &sp, int64_t n, std::vector<uint64_t> *cnt) {
        check(cudaMemsetAsync(S.cnt, 0, kContexts * kMaxAlphabet * 8, st));
        check(cudaMemsetAsync(S.extra, 0, 8, st));
        token_kernel<<<blocks_for(8 * n, 256), 256, 0, st>>>(S.ctx, S.val, n, sp, S.cnt, S.extra);
        check(cudaGetLastError());
        std::vector<unsigned long long> h(kContexts * kMaxAlphabet + 1);
        d2h(h.data(), S.cnt, kContexts * kMaxAlphabet);
        unsigned long long extra = 0;
        d2h(&extra, S.extra, 1);
        for (int c = 0; c < kContexts; ++c) {
            cnt[c].assign(split_alphabet(sp.m[c], kCtxLow[c]), 0);
            for (size_t t = 0; t < cnt[c].size(); ++t) cnt[c][t] = h[size_t(c) * kMaxAlphabet + t];
        }
        return extra;
    }

    double estimate(int k) {
        int64_t step = std::max<int64_t>(1, (P.nb + kSampleBlocks - 1) / kSampleBlocks);
        int64_t ns = (P.nb + step - 1) / step;
        Splits sp = quantize(k, step, ns);
        std::vector<uint64_t> cnt[kContexts];
        uint64_t extra = tokens(sp, ns, cnt);
        return estimate_from_counts(cnt, sp.m, P.coding, extra, P.nb, ns, P.rows, P.cols, P.container, P.T);
    }
};

}  // namespace
}  // namespace ep

extern "C" size_t ep_compress_device_scratch(int64_t rows, int64_t cols, const ep_config *cfg) {
    using namespace ep;
    if (rows <= 0 || cols <= 0 || !cfg) return 0;
    Plan P = plan_of(rows, cols, EP_BF16, cfg);
    if (!P.ok) return 0;
    // the code matrix is carved for every container so that the size does not depend on it
    return carve(nullptr, rows, cols, EP_INT8, P.nb, P.T).bytes;
}

extern "C" int ep_compress_device(const void *d_src, int32_t src_dtype, int64_t rows, int64_t cols,
                                  const ep_config *cfg, void *d_out, size_t out_cap, size_t *out_nbytes,
                                  void *d_scratch, size_t scratch_nbytes, ep_stream_t stream) {
    using namespace ep;
    if (!d_src || !cfg || !out_nbytes || !d_scratch || rows <= 0 || cols <= 0) return EP_ERR_INVALID_ARG;
    *out_nbytes = 0;
    if (!little_endian_host()) return EP_ERR_UNSUPPORTED;
    if (src_dtype != EP_BF16 && src_dtype != EP_FP16 && src_dtype != EP_FP32) return EP_ERR_UNSUPPORTED;
    int container = cfg->container_dtype ? cfg->container_dtype : src_dtype;
    if (container < EP_BF16 || container > EP_FP8_E4M3) return EP_ERR_INVALID_ARG;
    if (cfg->blocks_per_lane > 4096) return EP_ERR_INVALID_ARG;
    if (cfg->coding < EP_CODING_AUTO || cfg->coding > EP_CODING_PAIRED) return EP_ERR_INVALID_ARG;
    if ((rows * ((cols + 7) / 8)) >> 32) return EP_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(d_scratch) & 255u || reinterpret_cast<uintptr_t>(d_out) & 15u)
        return EP_ERR_INVALID_ARG;
    Plan P = plan_of(rows, cols, src_dtype, cfg);
    // P.ok is false for an unknown layout and for a shape or tile size the GEMM block order cannot take
    if (!P.ok || scratch_nbytes < ep_compress_device_scratch(rows, cols, cfg)) return EP_ERR_INVALID_ARG;
    int device = 0, sms = 0;
    if (cudaGetDevice(&device) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
        return EP_ERR_CUDA;
    Run R{P, DevSrc{d_src, src_dtype}, carve(static_cast<uint8_t *>(d_scratch), rows, cols, container, P.nb, P.T),
          reinterpret_cast<cudaStream_t>(stream), sms * 8};

    // rows: finite check, codes, scales, RMS
    R.check(cudaMemsetAsync(R.S.bad, 0, 4, R.st));
    rows_kernel<<<int((rows + 32 * kRowWarps - 1) / (32 * kRowWarps)), 32 * kRowWarps, 0, R.st>>>(
        R.src, rows, cols, container, R.S.codes, R.S.scales, R.S.rms, R.S.bad);
    R.check(cudaGetLastError());
    uint32_t bad = 0;
    R.d2h(&bad, R.S.bad, 1);
    if (R.err != cudaSuccess) return EP_ERR_CUDA;
    if (bad) return EP_ERR_NONFINITE;
    const double target = cfg->target_bpp;
    if (!(target >= 0.001) || !(target <= 11.0) || (is_code_container(container) && !(target < 8.0)))
        return EP_ERR_TARGET_RANGE;
    std::vector<float> rms(static_cast<size_t>(rows)), scales;
    R.d2h(rms.data(), R.S.rms, rms.size());
    if (is_code_container(container)) {
        scales.resize(size_t(rows));
        R.d2h(scales.data(), R.S.scales, scales.size());
    }

    // resolution: bisection on the sampled estimate (as the host compressor)
    const int kmax = max_q_index(cols);
    int k;
    if (cfg->q_index >= 0) {
        k = std::min(cfg->q_index, kmax);
    } else {
        const double budget = kTargetMargin * target;
        int lo = 0, hi = kmax;
        while (lo < hi && R.err == cudaSuccess) {
            int mid = lo + (hi - lo + 1) / 2;
            if (R.estimate(mid) <= budget)
                lo = mid;
            else
                hi = mid - 1;
        }
        k = lo;
    }

    // full encode at k; one resolution step down while the stream is over the target
    std::vector<uint32_t> count(size_t(P.T) * 32), dir(size_t(P.T) + 1);
    for (;;) {
        if (R.err != cudaSuccess) return EP_ERR_CUDA;
        Splits sp = R.quantize(k, 1, P.nb);
        std::vector<uint64_t> cnt[kContexts];
        R.tokens(sp, P.nb, cnt);
        std::vector<uint32_t> freq[kContexts];
        std::vector<uint8_t> rare;
        uint32_t ntok[kContexts], tablen[kContexts], A[kContexts] = {};
        uint64_t tokens = 0;
        const bool paired = pair_eligible(P.coding, P.nb, sp.m, cnt[1], cnt[2]);
        std::vector<unsigned long long> pc;
        if (paired) {
            A[1] = seen_len(cnt[1]);
            A[2] = seen_len(cnt[2]);
            R.check(cudaMemsetAsync(R.S.pairs, 0, 2 * kPairBins * 8, R.st));
            pair_kernel<<<R.blocks_for(P.nb, 256), 256, 0, R.st>>>(R.S.ctx, R.S.val, P.nb, sp, pair_base(A[1]),
                                                                   pair_base(A[2]), R.S.pairs);
            R.check(cudaGetLastError());
            pc.resize(2 * kPairBins);
            R.d2h(pc.data(), R.S.pairs, pc.size());
        }
        std::vector<uint16_t> hf(kContexts * kTableStride, 0), hc(kContexts * kTableStride, 0);
        for (int c = 0; c < kContexts; ++c) {
            if (paired && (c == 1 || c == 2)) {
                std::vector<uint64_t> pair_cnt(size_t(pair_base(A[c])) * pair_base(A[c]));
                for (size_t q = 0; q < pair_cnt.size(); ++q) pair_cnt[q] = pc[size_t(c - 1) * kPairBins + q];
                uint64_t N = 0;  // every token of the context belongs to one of its pairs
                for (uint64_t x : cnt[c]) N += x;
                build_pair_table(pair_cnt, A[c], N / 2, freq[c], rare);
                ntok[c] = A[c];
                tablen[c] = pair_table_len(A[c]);
            } else {
                ntok[c] = build_freqs(cnt[c], freq[c]);
                tablen[c] = ntok[c];
            }
            tokens += tablen[c];
            uint32_t a = 0;
            for (size_t t = 0; t < tablen[c]; ++t) {
                hf[size_t(c) * kTableStride + t] = uint16_t(freq[c][t]);
                hc[size_t(c) * kTableStride + t] = uint16_t(a);
                a += freq[c][t];
            }
        }
        R.h2d(R.S.freq, hf.data(), hf.size());
        R.h2d(R.S.cum, hc.data(), hc.size());
        R.check(cudaMemsetAsync(R.S.too_long, 0, 4, R.st));
        LaneArgs la{R.S.ctx, R.S.val, R.S.freq, R.S.cum, R.S.count, R.S.rwords, R.S.state, R.S.too_long,
                    R.S.dir, nullptr, P.nb, P.K, P.T, P.cb, P.layout, sp, paired ? 1u : 0u, {}, {}};
        for (int c = 0; c < kContexts; ++c) {
            la.B[c] = pair_base(A[c]);
            la.rawb[c] = pair_raw_bits(A[c]);
        }
        const int lane_blocks = int((uint64_t(P.T) * 32 + 255) / 256);
        lane_kernel<false><<<lane_blocks, 256, 0, R.st>>>(la);
        R.check(cudaGetLastError());
        uint32_t too_long = 0;
        R.d2h(&too_long, R.S.too_long, 1);
        R.d2h(count.data(), R.S.count, count.size());
        if (R.err != cudaSuccess) return EP_ERR_CUDA;
        if (too_long) return EP_ERR_UNSUPPORTED;  // a lane region beyond 65535 words (forced tile size)
        Layout L = layout_for(rows, container, tokens, P.T);
        uint64_t at = 0;
        for (uint32_t t = 0; t < P.T; ++t) {
            uint64_t words = 0;
            for (int l = 0; l < 32; ++l) words += count[size_t(t) * 32 + l];
            dir[t] = uint32_t(at);
            at += align16(kTileHead + 2 * words) / 16;
        }
        dir[P.T] = uint32_t(at);
        const size_t total = L.tiles + size_t(at) * 16;
        if (cfg->q_index < 0 && 8.0 * double(total) > target * double(rows * cols)) {
            if (k == 0) {
                *out_nbytes = total;
                return EP_ERR_TARGET_UNREACHABLE;
            }
            --k;
            continue;
        }
        *out_nbytes = total;
        if (!d_out || total > out_cap) return EP_ERR_BUFFER_TOO_SMALL;
        // header, factors, scales, tables, directory from the host; tiles from the lanes
        std::vector<uint8_t> front(L.tiles, 0);
        std::vector<float> fac(static_cast<size_t>(rows));
        for (int64_t r = 0; r < rows; ++r) fac[size_t(r)] = factor_of(rms[size_t(r)], k);
        uint32_t mm[kContexts];
        for (int c = 0; c < kContexts; ++c) mm[c] = sp.m[c];
        write_front(front.data(), L, src_dtype, container, rows, cols, P.T, P.K, k, mm, ntok, tablen, paired, freq,
                    fac.data(), scales.data(), P.layout);
        for (uint32_t t = 0; t <= P.T; ++t)
            for (int b = 0; b < 4; ++b) front[L.dir + 4 * t + b] = uint8_t(dir[t] >> (8 * b));
        uint8_t *out = static_cast<uint8_t *>(d_out);
        R.h2d(out, front.data(), front.size());
        R.check(cudaMemsetAsync(out + L.tiles, 0, total - L.tiles, R.st));
        R.h2d(R.S.dir, dir.data(), dir.size());
        la.tiles = out + L.tiles;
        lane_kernel<true><<<lane_blocks, 256, 0, R.st>>>(la);
        R.check(cudaGetLastError());
        R.check(cudaStreamSynchronize(R.st));  // the host buffers above must outlive the copies
        return R.err == cudaSuccess ? EP_OK : EP_ERR_CUDA;
    }
}
