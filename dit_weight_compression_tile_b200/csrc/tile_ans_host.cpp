// Tile-ANS host compressor and parser: ep_ans_compress_bound, ep_ans_compress_host and
// ep_ans_stream_info ("EntroPack README", Configuration: TileANSConfig, lossless compression for
// BF16, FP16, FP32, FP8 and INT8 tensors).  The stream layout is in tile_ans.h.  The compressor
// counts the elements' top bytes, turns the counts into a 12-bit table with the lattice stream's
// largest-remainder rule, and encodes the tiles' lanes on host threads, each lane's symbols in
// reverse decode order; the raw plane is the elements' low bytes copied in order.
#include <algorithm>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

#include "../../include/eptile.h"
#include "encode_host.h"
#include "tile_ans.h"

namespace ep {
namespace ta {
namespace {

void put(uint8_t *p, uint64_t v, int n) {
    for (int i = 0; i < n; ++i) p[i] = uint8_t(v >> (8 * i));
}
uint64_t rd(const uint8_t *p, int n) {
    uint64_t v = 0;
    for (int i = 0; i < n; ++i) v |= uint64_t(p[i]) << (8 * i);
    return v;
}

void parallel_for(int64_t n, int threads, const std::function<void(int64_t, int64_t)> &fn) {
    if (n <= 0) return;
    int64_t nt = std::max<int64_t>(1, std::min<int64_t>(threads, n));
    if (nt == 1) {
        fn(0, n);
        return;
    }
    std::vector<std::thread> pool;
    int64_t chunk = (n + nt - 1) / nt;
    for (int64_t t = 0; t < nt; ++t) {
        int64_t b = t * chunk, e = std::min(n, b + chunk);
        if (b < e) pool.emplace_back(fn, b, e);
    }
    for (auto &th : pool) th.join();
}

int hw_threads(int asked) {
    if (asked > 0) return asked;
    unsigned h = std::thread::hardware_concurrency();
    return h ? int(h) : 1;
}

}  // namespace
}  // namespace ta
}  // namespace ep

extern "C" size_t ep_ans_compress_bound(int64_t n, int32_t dtype) {
    using namespace ep::ta;
    const int esz = elt_bytes(dtype);
    if (n <= 0 || esz == 0) return 0;
    const int64_t nc = (n + kChunk - 1) / kChunk;
    // every symbol costs at most 12 + 1 bits (a word per symbol at worst); tiles of the smallest
    // automatic size; heads, padding and the sections in front
    const uint64_t tiles = uint64_t((nc + kLanes * 16 - 1) / (kLanes * 16)) + 1;
    const Layout L = layout_for(n, esz, tiles);
    return L.tiles + size_t(nc) * kChunk * 2 + tiles * (kTileHead + 16) + 64;
}

extern "C" int ep_ans_compress_host(const void *srcv, int64_t n, int32_t ndim, const int64_t *shape,
                                    const ep_ans_config *cfg, void *outv, size_t out_cap, size_t *out_nbytes) {
    using namespace ep::ta;
    if (!srcv || !cfg || !out_nbytes || n <= 0 || ndim < 1 || ndim > kMaxDims || !shape) return EP_ERR_INVALID_ARG;
    const int esz = elt_bytes(cfg->dtype);
    if (esz == 0) return EP_ERR_INVALID_ARG;
    int64_t prod = 1;
    for (int d = 0; d < ndim; ++d) {
        if (shape[d] <= 0 || shape[d] > n) return EP_ERR_INVALID_ARG;
        prod *= shape[d];
        if (prod > n) return EP_ERR_INVALID_ARG;
    }
    if (prod != n) return EP_ERR_INVALID_ARG;
    const uint8_t *src = static_cast<const uint8_t *>(srcv);
    const int64_t nc = (n + kChunk - 1) / kChunk;
    const uint32_t K = cfg->blocks_per_lane ? cfg->blocks_per_lane : auto_blocks_per_lane(nc);
    if (K > 4096) return EP_ERR_INVALID_ARG;
    const int64_t per_tile = int64_t(kLanes) * K;
    const int64_t T64 = (nc + per_tile - 1) / per_tile;
    if (T64 >= (int64_t(1) << 32)) return EP_ERR_UNSUPPORTED;
    const uint32_t T = uint32_t(T64);
    const int threads = hw_threads(cfg->n_threads);
    auto sym = [&](int64_t i) -> uint32_t { return i < n ? src[i * esz + (esz - 1)] : 0u; };

    // symbol counts over every chunk (the last one's zero padding included)
    std::vector<std::vector<uint64_t>> part(size_t(threads), std::vector<uint64_t>(256, 0));
    const int64_t nsym = nc * kChunk;
    {
        const int64_t per = (nsym + threads - 1) / threads;
        std::vector<std::thread> pool;
        for (int t = 0; t < threads; ++t) {
            const int64_t b = int64_t(t) * per, e = std::min(nsym, b + per);
            if (b >= e) break;
            pool.emplace_back([&, t, b, e] {
                auto &h = part[size_t(t)];
                for (int64_t i = b; i < e; ++i) ++h[sym(i)];
            });
        }
        for (auto &th : pool) th.join();
    }
    std::vector<uint64_t> cnt(256, 0);
    for (auto &h : part)
        for (int s = 0; s < 256; ++s) cnt[size_t(s)] += h[size_t(s)];
    std::vector<uint32_t> f;
    ep::build_freqs(cnt, f, kProbScale);
    uint32_t cum[257];
    cum[0] = 0;
    for (int s = 0; s < 256; ++s) cum[s + 1] = cum[s] + f[size_t(s)];

    // every lane's words (reverse decode order, then reversed) and final state
    const size_t maxw = size_t(K) * kChunk + 4;
    std::vector<uint16_t> words(size_t(T) * kLanes * maxw);
    std::vector<uint32_t> nw(size_t(T) * kLanes), state(size_t(T) * kLanes);
    std::vector<uint64_t> tile_bytes(T);
    bool too_long = false;
    parallel_for(T, threads, [&](int64_t t0, int64_t t1) {
        for (int64_t t = t0; t < t1; ++t) {
            uint64_t tw = 0;
            for (int l = 0; l < kLanes; ++l) {
                uint16_t *w = words.data() + (size_t(t) * kLanes + l) * maxw;
                uint32_t m = 0, x = kStateLow;
                for (int64_t k = int64_t(K) - 1; k >= 0; --k) {
                    const int64_t c = t * per_tile + k * kLanes + l;
                    if (c >= nc) continue;
                    for (int j = kChunk - 1; j >= 0; --j) {
                        const uint32_t s = sym(c * kChunk + j), fs = f[s];
                        if (x >= (fs << 20)) {  // keeps the state in [2^16, 2^32) after the update
                            w[m++] = uint16_t(x & 0xffffu);
                            x >>= 16;
                        }
                        x = ((x / fs) << kProbBits) + (x % fs) + cum[s];
                    }
                }
                std::reverse(w, w + m);
                if (m > 0xffffu) too_long = true;
                nw[size_t(t) * kLanes + l] = m;
                state[size_t(t) * kLanes + l] = x;
                tw += m;
            }
            tile_bytes[size_t(t)] = align16(kTileHead + 2 * tw);
        }
    });
    if (too_long) return EP_ERR_UNSUPPORTED;
    std::vector<uint32_t> toff(size_t(T) + 1);
    uint64_t acc = 0;
    for (uint32_t t = 0; t < T; ++t) {
        if (acc / 16 >= (uint64_t(1) << 32)) return EP_ERR_UNSUPPORTED;
        toff[t] = uint32_t(acc / 16);
        acc += tile_bytes[t];
    }
    if (acc / 16 >= (uint64_t(1) << 32)) return EP_ERR_UNSUPPORTED;
    toff[T] = uint32_t(acc / 16);
    const Layout L = layout_for(n, esz, T);
    const size_t total = L.tiles + size_t(acc);
    *out_nbytes = total;
    if (!outv || out_cap < total) return EP_ERR_BUFFER_TOO_SMALL;
    uint8_t *out = static_cast<uint8_t *>(outv);
    std::memset(out, 0, L.tiles);
    put(out, kMagic, 4);
    put(out + 4, kVersion, 2);
    out[6] = uint8_t(cfg->dtype);
    out[7] = uint8_t(ndim);
    put(out + 8, uint64_t(n), 8);
    put(out + 16, T, 4);
    put(out + 20, K, 4);
    out[24] = uint8_t(kProbBits);
    for (int d = 0; d < ndim; ++d) put(out + kHeaderBytes + 8 * d, uint64_t(shape[d]), 8);
    for (int s = 0; s < 256; ++s) put(out + L.freq + 2 * s, f[size_t(s)], 2);
    for (uint32_t t = 0; t <= T; ++t) put(out + L.dir + 4 * t, toff[t], 4);
    // the raw plane: each element's low bytes, in element order
    if (esz > 1) {
        uint8_t *raw = out + L.raw;
        parallel_for(n, threads, [&](int64_t i0, int64_t i1) {
            for (int64_t i = i0; i < i1; ++i) std::memcpy(raw + i * (esz - 1), src + i * esz, size_t(esz - 1));
        });
    }
    parallel_for(T, threads, [&](int64_t t0, int64_t t1) {
        for (int64_t t = t0; t < t1; ++t) {
            uint8_t *tp = out + L.tiles + 16 * size_t(toff[size_t(t)]);
            std::memset(tp, 0, tile_bytes[size_t(t)]);
            size_t pos = kTileHead;
            for (int l = 0; l < kLanes; ++l) {
                const size_t li = size_t(t) * kLanes + l;
                put(tp + 4 * l, state[li], 4);
                put(tp + 128 + 2 * l, nw[li], 2);
                const uint16_t *w = words.data() + li * maxw;
                for (uint32_t a = 0; a < nw[li]; ++a, pos += 2) put(tp + pos, w[a], 2);
            }
        }
    });
    return EP_OK;
}

extern "C" int ep_ans_stream_info(const void *blob, size_t nbytes, ep_ans_info *info) {
    using namespace ep::ta;
    if (!blob || !info) return EP_ERR_INVALID_ARG;
    const uint8_t *p = static_cast<const uint8_t *>(blob);
    if (nbytes < kHeaderBytes + 8 * kMaxDims + 512) return EP_ERR_CORRUPT;
    ep_ans_info I;
    std::memset(&I, 0, sizeof I);
    if (rd(p, 4) != kMagic || rd(p + 4, 2) != kVersion || p[24] != kProbBits) return EP_ERR_CORRUPT;
    I.dtype = p[6];
    I.ndim = p[7];
    I.n_elems = int64_t(rd(p + 8, 8));
    I.n_tiles = uint32_t(rd(p + 16, 4));
    I.blocks_per_lane = uint32_t(rd(p + 20, 4));
    const int esz = elt_bytes(I.dtype);
    if (esz == 0 || I.ndim < 1 || I.ndim > kMaxDims || I.n_elems <= 0 || I.n_elems >= (int64_t(1) << 40) ||
        I.blocks_per_lane < 1 || I.blocks_per_lane > 4096)
        return EP_ERR_CORRUPT;
    int64_t prod = 1;
    for (int d = 0; d < I.ndim; ++d) {
        I.shape[d] = int64_t(rd(p + kHeaderBytes + 8 * d, 8));
        if (I.shape[d] <= 0 || I.shape[d] > I.n_elems) return EP_ERR_CORRUPT;
        prod *= I.shape[d];
        if (prod > I.n_elems) return EP_ERR_CORRUPT;
    }
    if (prod != I.n_elems) return EP_ERR_CORRUPT;
    const int64_t nc = (I.n_elems + kChunk - 1) / kChunk, per_tile = int64_t(kLanes) * I.blocks_per_lane;
    if ((nc + per_tile - 1) / per_tile != int64_t(I.n_tiles)) return EP_ERR_CORRUPT;
    const Layout L = layout_for(I.n_elems, esz, I.n_tiles);
    if (L.tiles > nbytes) return EP_ERR_CORRUPT;
    uint32_t sum = 0;
    for (int s = 0; s < 256; ++s) {
        const uint32_t fs = uint32_t(rd(p + L.freq + 2 * s, 2));
        if (fs >= kProbScale) return EP_ERR_CORRUPT;  // the slot entry holds 12 bits of it
        sum += fs;
    }
    if (sum != kProbScale) return EP_ERR_CORRUPT;
    uint64_t prev = rd(p + L.dir, 4), largest = 0;
    if (prev != 0) return EP_ERR_CORRUPT;
    for (uint32_t t = 1; t <= I.n_tiles; ++t) {
        const uint64_t cur = rd(p + L.dir + 4 * t, 4);
        if (cur < prev + kTileHead / 16) return EP_ERR_CORRUPT;
        largest = std::max(largest, cur - prev);
        prev = cur;
    }
    if (L.tiles + 16 * prev != nbytes) return EP_ERR_CORRUPT;
    I.storage_nbytes = nbytes;
    I.out_nbytes = uint64_t(I.n_elems) * uint64_t(esz);
    I.ratio = double(nbytes) / double(I.out_nbytes);
    I.off_freq = L.freq;
    I.off_dir = L.dir;
    I.off_raw = L.raw;
    I.off_tiles = L.tiles;
    I.max_tile_nbytes = 16 * largest;
    I.workspace_nbytes = kTableBytes;
    *info = I;
    return EP_OK;
}
