// Host compressor: ep_compress_host / ep_compress_bound.
//
// compress(tensor, config) of the "EntroPack API reference", following the pipeline of the
// "EntroPack: Fast and Accurate Entropy-Coded Weight Compression at Arbitrary Bitrates"
// Abstract: row-normalized E8 lattice quantization, a conditional model of the lattice
// coordinates, a resolution picked by sampled storage estimates (no repeated full-stream
// encoding in the normal case), and entropy coding in tiles that decode on their own.
// Multithreaded over rows, blocks and tiles; the output bytes do not depend on the thread
// count (every floating-point reduction keeps a fixed order).
#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

#include "../../include/eptile.h"
#include "encode_host.h"
#include "encode_math.h"
#include "format.h"

namespace ep {
namespace {

// ------------------------------------------------------------------ threading
void parallel_for(int64_t n, int threads, const std::function<void(int64_t, int64_t)> &fn) {
    if (n <= 0) return;
    int64_t nt = std::max<int64_t>(1, std::min<int64_t>(threads, (n + 1023) / 1024));
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

// ------------------------------------------------------------------ source values
// fp16 -> float through a table built from the bit fields (exact)
const float *half_table() {
    static std::vector<float> tab = [] {
        std::vector<float> t(65536);
        for (uint32_t h = 0; h < 65536; ++h) {
            uint32_t sign = (h & 0x8000u) << 16, exp = (h >> 10) & 31, man = h & 1023;
            float v;
            if (exp == 0) {
                v = std::ldexp(float(man), -24);
            } else if (exp == 31) {
                v = man ? NAN : INFINITY;
            } else {
                v = std::ldexp(float(man | 1024u), int(exp) - 25);
            }
            uint32_t b;
            std::memcpy(&b, &v, 4);
            b |= sign;
            std::memcpy(&v, &b, 4);
            t[h] = v;
        }
        return t;
    }();
    return tab.data();
}

struct Source {
    const void *p;
    int dt;
    float at(int64_t i) const {
        if (dt == EP_BF16) {
            uint32_t b = uint32_t(static_cast<const uint16_t *>(p)[i]) << 16;
            float f;
            std::memcpy(&f, &b, 4);
            return f;
        }
        if (dt == EP_FP16) return half_table()[static_cast<const uint16_t *>(p)[i]];
        return static_cast<const float *>(p)[i];
    }
};

}  // namespace

// ------------------------------------------------------------------ decisions from histograms
int max_q_index(int64_t cols) {
    double lim = std::ldexp(1.0, 20) / (std::sqrt(double(cols)) + 1.0);
    int k = kNumQ - 1;
    while (k > 0 && q_value(k) > lim) --k;
    return k;
}

// smallest m allowed for the context with >= 99.9% of the values below 2^m (bit length <= m)
uint32_t pick_split(const uint64_t *by_len, int ctx) {
    uint32_t lo = kTopBits + kCtxLow[ctx], hi = kCtxMaxSplit[ctx];
    uint64_t n = 0;
    for (int i = 0; i <= 32; ++i) n += by_len[i];
    if (!n) return lo;
    uint64_t acc = 0;
    for (uint32_t m = 0; m <= hi; ++m) {
        acc += by_len[m];
        if (m >= lo && acc * 1000u >= n * 999u) return m;
    }
    return hi;
}

// largest remainders to a sum of `scale` (2^11 for token tables, 2^12 for pair tables), then
// every seen symbol raised to >= 1 from the currently largest frequency (lowest index on ties);
// a lone seen symbol keeps scale - 1 and gives one unit to a phantom symbol (1 if it is 0, else 0)
uint32_t build_freqs(const std::vector<uint64_t> &cnt, std::vector<uint32_t> &f, uint32_t scale) {
    size_t n = cnt.size();
    f.assign(n, 0);
    uint64_t total = 0;
    uint32_t len = 0, seen = 0, only = 0;
    for (size_t i = 0; i < n; ++i) {
        total += cnt[i];
        if (cnt[i]) {
            len = uint32_t(i + 1);
            ++seen;
            only = uint32_t(i);
        }
    }
    if (!total) return 0;
    if (seen == 1) {
        uint32_t phantom = only == 0 ? 1u : 0u;
        f[only] = scale - 1;
        f[phantom] = 1;
        return std::max(len, phantom + 1);
    }
    std::vector<std::pair<uint64_t, uint32_t>> rems;  // (remainder, index)
    uint32_t used = 0;
    for (size_t i = 0; i < n; ++i) {
        if (!cnt[i]) continue;
        uint64_t scaled = cnt[i] * scale;
        f[i] = uint32_t(scaled / total);
        used += f[i];
        rems.emplace_back(scaled % total, uint32_t(i));
    }
    std::stable_sort(rems.begin(), rems.end(),
                     [](const auto &a, const auto &b) { return a.first > b.first; });
    for (uint32_t r = 0; r < scale - used; ++r) f[rems[r].second] += 1;
    for (size_t i = 0; i < n; ++i) {
        if (cnt[i] && !f[i]) {
            size_t big = size_t(std::max_element(f.begin(), f.end()) - f.begin());
            f[big] -= 1;
            f[i] = 1;
        }
    }
    return len;
}

uint32_t seen_len(const std::vector<uint64_t> &cnt) {
    uint32_t len = 0;
    for (size_t t = 0; t < cnt.size(); ++t)
        if (cnt[t]) len = uint32_t(t + 1);
    return len;
}

// pairs when asked to (EP_CODING_PAIRED) or, automatically, from 2^17 blocks on; in both cases
// only with splits that keep every coordinate in [-256, 255], alphabets of contexts 1 and 2 of at
// most 256 tokens and at most 1 / 2^12 of their tokens at or beyond the base
bool pair_eligible(int coding, int64_t nb, const uint32_t *m, const std::vector<uint64_t> &cnt1,
                   const std::vector<uint64_t> &cnt2) {
    if (coding == EP_CODING_SINGLE) return false;
    for (int c = 0; c < kContexts; ++c)
        if (m[c] > kCtxNarrowSplit[c]) return false;
    for (const std::vector<uint64_t> *cnt : {&cnt1, &cnt2}) {
        uint64_t all = 0, outside = 0;
        for (size_t t = 0; t < cnt->size(); ++t) {
            all += (*cnt)[t];
            if (t >= kPairBaseMax) outside += (*cnt)[t];
        }
        if (seen_len(*cnt) > kPairMaxAlphabet || outside * kPairOutsideScale > all) return false;
    }
    return coding == EP_CODING_PAIRED || nb >= kPairMinBlocks;
}

void build_pair_table(std::vector<uint64_t> pair_cnt, uint32_t A, uint64_t N, std::vector<uint32_t> &f,
                      std::vector<uint8_t> &rare) {
    const uint32_t n = pair_table_len(A);
    pair_cnt.resize(n, 0);
    rare.assign(n, 0);
    f.assign(n, 0);
    if (!n) return;
    uint64_t inside = 0;
    for (uint32_t q = 0; q + 1 < n; ++q) inside += pair_cnt[q];
    pair_cnt[n - 1] = N - inside;  // pairs with a token outside the base
    for (uint32_t q = 0; q + 1 < n; ++q)
        if (pair_cnt[q] && pair_cnt[q] * kPairRareScale < N) {
            rare[q] = 1;
            pair_cnt[n - 1] += pair_cnt[q];
            pair_cnt[q] = 0;
        }
    build_freqs(pair_cnt, f, kPairScale);
}

double estimate_from_counts(const std::vector<uint64_t> *cnt, const uint32_t *m, int coding, uint64_t extra_bits,
                            int64_t nb, int64_t ns, int64_t rows, int64_t cols, int container, uint32_t T) {
    double bits = 0.0;
    uint64_t tokens = 0;
    // a paired stream stores pair tables for contexts 1 and 2; its payload is estimated by the
    // same token entropy
    const bool paired = pair_eligible(coding, nb, m, cnt[1], cnt[2]);
    for (int c = 0; c < kContexts; ++c) {
        uint64_t n = 0;
        for (size_t t = 0; t < cnt[c].size(); ++t) n += cnt[c][t];
        const uint32_t len = seen_len(cnt[c]);
        tokens += paired && (c == 1 || c == 2) ? pair_table_len(len) : len;
        if (!n) continue;
        bits += double(n) * std::log2(double(n));
        for (size_t t = 0; t < cnt[c].size(); ++t)
            if (cnt[c][t]) bits -= double(cnt[c][t]) * std::log2(double(cnt[c][t]));
    }
    bits += double(extra_bits);
    Layout L = layout_for(rows, container, tokens, T);
    double bytes = double(L.tiles) + kTileOverheadBytes * double(T) + bits * (double(nb) / double(ns)) / 8.0;
    return 8.0 * bytes / double(rows * cols);
}

void write_front(uint8_t *h, const Layout &L, int src_dt, int container, int64_t rows, int64_t cols, uint32_t T,
                 uint32_t K, int k, const uint32_t *m, const uint32_t *ntok, const uint32_t *tablen, bool paired,
                 const std::vector<uint32_t> *freq, const float *fac, const float *scales, int layout) {
    auto put = [](uint8_t *p, uint64_t v, int n) {
        for (int i = 0; i < n; ++i) p[i] = uint8_t(v >> (8 * i));
    };
    put(h, kMagic, 4);
    put(h + 4, kVersion, 2);
    h[6] = uint8_t(src_dt);
    h[7] = uint8_t(container);
    put(h + 8, uint64_t(rows), 8);
    put(h + 16, uint64_t(cols), 8);
    put(h + 24, T, 4);
    put(h + 28, K, 4);
    put(h + 32, uint32_t(k), 2);
    h[34] = uint8_t(kProbBits);
    h[35] = uint8_t(kContexts);
    h[43] = paired ? 1 : 0;
    h[58] = uint8_t(layout);
    for (int c = 0; c < kContexts; ++c) {
        h[36 + c] = uint8_t(m[c]);
        put(h + 44 + 2 * c, ntok[c], 2);
    }
    std::memcpy(h + L.rowf, fac, size_t(rows) * 4);
    if (is_code_container(container)) std::memcpy(h + L.scales, scales, size_t(rows) * 4);
    size_t q = L.freq;
    for (int c = 0; c < kContexts; ++c)
        for (uint32_t t = 0; t < tablen[c]; ++t, q += 2) put(h + q, freq[c][t], 2);
}

bool little_endian_host() {
    uint32_t one = 1;
    uint8_t b;
    std::memcpy(&b, &one, 1);
    return b == 1;
}

namespace {

// ------------------------------------------------------------------ the encoder
struct Encoder {
    Source src;
    int64_t rows, cols, cb, nb;  // cb = ceil(cols / 8): a row is zero-padded to whole E8 blocks
    int container;
    int threads;
    int coding;  // EP_CODING_*
    int layout;  // EP_LAYOUT_*: the block order of the tiles
    uint32_t K;
    std::vector<float> codes;   // INT8/FP8 code matrix (exact in fp32), empty otherwise
    std::vector<float> scales;  // INT8/FP8 per-row scales
    std::vector<float> rms;     // per-row RMS s_r

    double value(int64_t i) const { return codes.empty() ? double(src.at(i)) : double(codes[size_t(i)]); }

    void quantize_block(int64_t b, float f, int32_t *v) const {
        if (f == 0.0f) {
            std::fill(v, v + 8, 0);
            return;
        }
        // block b holds columns c0 .. c0 + 7 of row r; columns past the row's end are zeros
        const int64_t r = b / cb, c0 = 8 * (b - r * cb), base = r * cols + c0;
        const int n8 = int(std::min<int64_t>(8, cols - c0));
        double x[8], two_f = 2.0 * double(f);
        for (int i = 0; i < 8; ++i) x[i] = i < n8 ? value(base + i) / two_f : 0.0;
        quantize_e8(x, v);
    }

    void prepare() {
        cb = (cols + 7) / 8;
        nb = rows * cb;
        if (is_code_container(container)) {
            codes.resize(size_t(rows * cols));
            scales.resize(size_t(rows));
            double bound = container == EP_INT8 ? 127.0 : 448.0;
            parallel_for(rows, threads, [&](int64_t r0, int64_t r1) {
                for (int64_t r = r0; r < r1; ++r) {
                    double amax = 0.0;
                    for (int64_t j = 0; j < cols; ++j) amax = std::max(amax, std::fabs(double(src.at(r * cols + j))));
                    float s = amax > 0.0 ? float(amax / bound) : 1.0f;
                    if (s == 0.0f) s = FLT_MIN;
                    scales[size_t(r)] = s;
                    for (int64_t j = 0; j < cols; ++j) {
                        double w = src.at(r * cols + j);
                        double c;
                        if (amax == 0.0) {
                            c = 0.0;
                        } else if (container == EP_INT8) {
                            c = std::min(127.0, std::max(-127.0, std::nearbyint(w / double(s))));
                        } else {
                            c = e4m3_round(float(w / double(s)));
                        }
                        codes[size_t(r * cols + j)] = float(c);
                    }
                }
            });
        }
        rms.resize(size_t(rows));
        parallel_for(rows, threads, [&](int64_t r0, int64_t r1) {
            for (int64_t r = r0; r < r1; ++r) {
                double acc = 0.0;
                for (int64_t j = 0; j < cols; ++j) {
                    double a = value(r * cols + j);
                    acc += a * a;
                }
                rms[size_t(r)] = float(std::sqrt(acc / double(cols)));
            }
        });
    }

    uint32_t tile_count() const { return uint32_t((nb + int64_t(kLanes) * K - 1) / (int64_t(kLanes) * K)); }

    // ---- sampled storage estimate (bits per weight at resolution index k)
    double estimate(int k) const {
        int64_t step = std::max<int64_t>(1, (nb + kSampleBlocks - 1) / kSampleBlocks);
        int64_t ns = (nb + step - 1) / step;
        std::vector<uint8_t> ctx(static_cast<size_t>(ns) * 8);
        std::vector<uint32_t> val(static_cast<size_t>(ns) * 8);
        parallel_for(ns, threads, [&](int64_t j0, int64_t j1) {
            for (int64_t j = j0; j < j1; ++j) {
                int64_t b = j * step;
                int32_t v[8];
                quantize_block(b, factor_of(rms[size_t(b / cb)], k), v);
                symbols_of(v, &ctx[size_t(8 * j)], &val[size_t(8 * j)]);
            }
        });
        uint64_t by_len[kContexts][33] = {};
        for (size_t i = 0; i < val.size(); ++i) by_len[ctx[i]][bitlen(val[i])]++;
        uint32_t m[kContexts];
        std::vector<uint64_t> cnt[kContexts];
        for (int c = 0; c < kContexts; ++c) {
            m[c] = pick_split(by_len[c], c);
            cnt[c].assign(split_alphabet(m[c], kCtxLow[c]), 0);
        }
        uint64_t extra = 0;
        for (size_t i = 0; i < val.size(); ++i) {
            Token t = token_of(val[i], m[ctx[i]], kCtxLow[ctx[i]]);
            cnt[ctx[i]][t.tok]++;
            extra += t.nbits;
        }
        return estimate_from_counts(cnt, m, coding, extra, nb, ns, rows, cols, container, tile_count());
    }

    // ---- one tile: 32 independent lanes.  A lane's region holds its rANS words in decode order
    // followed by its raw bits, packed least significant bit first into 16-bit words that are
    // stored back to front (the region's last word holds the first 16 raw bits).  Per block the
    // symbols are the 8 tokens (single coding) or token 0, the pair symbols of coordinates (1,2),
    // (3,4), (5,6) and token 7 (paired coding); the raw bits are the tokens of the escaped pairs
    // (paired coding), then the extra bits of coordinates 0..7.  Returns false when a region
    // exceeds 65535 words.
    struct Event {
        uint16_t f, cum;
        uint8_t bits;  // the symbol's table sums to 2^bits
    };
    struct Model {
        const uint32_t *m;
        const std::vector<uint32_t> *freq, *cum;  // paired contexts 1, 2: the pair tables
        bool paired;
        const uint32_t *A;                         // paired contexts 1, 2: token alphabet length
        const std::vector<uint8_t> *rare;          // paired contexts 1, 2: escaped pair indices
    };

    static bool encode_tile(const uint8_t *ctx, const uint32_t *val, int64_t nb, int64_t cb, int layout, int64_t t,
                            uint32_t K, const Model &M, std::vector<Event> &ev, std::vector<uint16_t> &words,
                            std::vector<uint8_t> &out) {
        uint32_t state[kLanes];
        uint32_t count[kLanes];
        bool fits = true;
        words.clear();
        for (int l = 0; l < kLanes; ++l) {
            ev.clear();
            size_t before = words.size();
            uint64_t acc = 0;
            uint32_t nacc = 0;
            std::vector<uint16_t> raw;
            auto add = [&](uint32_t c, uint32_t sym, uint32_t bits) {
                ev.push_back({uint16_t(M.freq[c][sym]), uint16_t(M.cum[c][sym]), uint8_t(bits)});
            };
            auto push = [&](uint32_t v, uint32_t nbits) {
                acc |= uint64_t(v) << nacc;
                nacc += nbits;
                while (nacc >= 16) {
                    raw.push_back(uint16_t(acc));
                    acc >>= 16;
                    nacc -= 16;
                }
            };
            for (uint32_t k = 0; k < K; ++k) {
                int64_t b = lane_block(layout, cb, t, l, K, k);
                if (b >= nb) break;
                const size_t s0 = size_t(8 * b);
                Token tk[8];
                for (int i = 0; i < 8; ++i) tk[i] = token_of(val[s0 + i], M.m[ctx[s0 + i]], kCtxLow[ctx[s0 + i]]);
                if (!M.paired) {
                    for (int i = 0; i < 8; ++i) add(ctx[s0 + i], tk[i].tok, kProbBits);
                } else {
                    const uint32_t pc = ctx[s0 + 1], A = M.A[pc], B = pair_base(A);
                    bool esc[3];
                    add(ctx[s0], tk[0].tok, kProbBits);
                    for (int j = 0; j < 3; ++j) {
                        const uint32_t ta = tk[1 + 2 * j].tok, tb = tk[2 + 2 * j].tok;
                        esc[j] = ta >= B || tb >= B || M.rare[pc][ta * B + tb] != 0;
                        add(pc, esc[j] ? B * B : ta * B + tb, kPairBits);
                    }
                    add(ctx[s0 + 7], tk[7].tok, kProbBits);
                    for (int j = 0; j < 3; ++j)
                        if (esc[j]) {
                            push(tk[1 + 2 * j].tok, pair_raw_bits(A));
                            push(tk[2 + 2 * j].tok, pair_raw_bits(A));
                        }
                }
                for (int i = 0; i < 8; ++i) push(tk[i].extra, tk[i].nbits);
            }
            if (nacc) raw.push_back(uint16_t(acc));
            uint32_t x = kStateLow;
            for (size_t e = ev.size(); e-- > 0;) {
                const uint32_t f = ev[e].f, n = ev[e].bits;
                if (uint64_t(x) >= (uint64_t(f) << (32 - n))) {  // keep the next state below 2^32
                    words.push_back(uint16_t(x));
                    x >>= 16;
                }
                x = (x / f) * (1u << n) + (x % f) + ev[e].cum;
            }
            std::reverse(words.begin() + long(before), words.end());  // decode order
            words.insert(words.end(), raw.rbegin(), raw.rend());
            state[l] = x;
            size_t n = words.size() - before;
            if (n > 0xffff) fits = false;
            count[l] = uint32_t(n);
        }
        size_t base = out.size();
        size_t bytes = align16(kTileHead + 2 * words.size());
        out.resize(base + bytes, 0);
        uint8_t *p = out.data() + base;
        for (int l = 0; l < kLanes; ++l) {
            for (int b = 0; b < 4; ++b) p[4 * l + b] = uint8_t(state[l] >> (8 * b));
            p[4 * kLanes + 2 * l] = uint8_t(count[l]);
            p[4 * kLanes + 2 * l + 1] = uint8_t(count[l] >> 8);
        }
        p += kTileHead;
        for (size_t i = 0; i < words.size(); ++i) {
            p[2 * i] = uint8_t(words[i]);
            p[2 * i + 1] = uint8_t(words[i] >> 8);
        }
        return fits;
    }

    // ---- full stream at resolution index k
    std::vector<uint8_t> encode(int k) const {
        std::vector<uint8_t> ctx(static_cast<size_t>(nb) * 8);
        std::vector<uint32_t> val(static_cast<size_t>(nb) * 8);
        std::vector<float> fac(static_cast<size_t>(rows));
        for (int64_t r = 0; r < rows; ++r) fac[size_t(r)] = factor_of(rms[size_t(r)], k);
        int nchunks = int(std::max<int64_t>(1, std::min<int64_t>(threads, (nb + 1023) / 1024)));
        std::vector<std::vector<uint64_t>> part_len(size_t(nchunks), std::vector<uint64_t>(kContexts * 33, 0));
        int64_t per = (nb + nchunks - 1) / nchunks;
        parallel_for(nchunks, nchunks, [&](int64_t c0, int64_t c1) {
            for (int64_t c = c0; c < c1; ++c) {
                auto &hist = part_len[size_t(c)];
                for (int64_t b = c * per; b < std::min(nb, (c + 1) * per); ++b) {
                    int32_t v[8];
                    quantize_block(b, fac[size_t(b / cb)], v);
                    symbols_of(v, &ctx[size_t(8 * b)], &val[size_t(8 * b)]);
                    for (int i = 0; i < 8; ++i) hist[size_t(ctx[size_t(8 * b + i)] * 33 + bitlen(val[size_t(8 * b + i)]))]++;
                }
            }
        });
        uint64_t by_len[kContexts][33] = {};
        for (auto &h : part_len)
            for (int c = 0; c < kContexts; ++c)
                for (int i = 0; i < 33; ++i) by_len[c][i] += h[size_t(c * 33 + i)];
        uint32_t m[kContexts];
        for (int c = 0; c < kContexts; ++c) m[c] = pick_split(by_len[c], c);
        // token counts
        std::vector<std::vector<uint64_t>> part_cnt(static_cast<size_t>(nchunks));
        parallel_for(nchunks, nchunks, [&](int64_t c0, int64_t c1) {
            for (int64_t c = c0; c < c1; ++c) {
                auto &cnt = part_cnt[size_t(c)];
                cnt.assign(kContexts * kMaxAlphabet, 0);
                for (int64_t s = 8 * c * per; s < 8 * std::min(nb, (c + 1) * per); ++s) {
                    uint8_t cx = ctx[size_t(s)];
                    cnt[size_t(cx) * kMaxAlphabet + token_of(val[size_t(s)], m[cx], kCtxLow[cx]).tok]++;
                }
            }
        });
        std::vector<uint32_t> freq[kContexts], cum[kContexts];
        std::vector<uint8_t> rare[kContexts];
        uint32_t ntok[kContexts], tablen[kContexts], A[kContexts] = {};
        uint64_t tokens = 0;
        std::vector<uint64_t> cnt[kContexts];
        for (int c = 0; c < kContexts; ++c) {
            cnt[c].assign(split_alphabet(m[c], kCtxLow[c]), 0);
            for (auto &pc : part_cnt)
                for (size_t t = 0; t < cnt[c].size(); ++t) cnt[c][t] += pc[size_t(c) * kMaxAlphabet + t];
        }
        const bool paired = pair_eligible(coding, nb, m, cnt[1], cnt[2]);
        for (int c = 0; c < kContexts; ++c) {
            if (paired && (c == 1 || c == 2)) {
                // counts of the token pairs of coordinates (1,2), (3,4), (5,6) inside the base
                A[c] = seen_len(cnt[c]);
                const uint32_t B = pair_base(A[c]), a2 = B * B;
                std::vector<std::vector<uint64_t>> part_pair(static_cast<size_t>(nchunks));
                parallel_for(nchunks, nchunks, [&](int64_t c0, int64_t c1) {
                    for (int64_t q = c0; q < c1; ++q) {
                        auto &pp = part_pair[size_t(q)];
                        pp.assign(a2, 0);
                        for (int64_t b = q * per; b < std::min(nb, (q + 1) * per); ++b) {
                            if (ctx[size_t(8 * b + 1)] != c) continue;
                            for (int j = 0; j < 3; ++j) {
                                uint32_t ta = token_of(val[size_t(8 * b + 1 + 2 * j)], m[c], kCtxLow[c]).tok;
                                uint32_t tb = token_of(val[size_t(8 * b + 2 + 2 * j)], m[c], kCtxLow[c]).tok;
                                if (ta < B && tb < B) pp[ta * B + tb]++;
                            }
                        }
                    }
                });
                std::vector<uint64_t> pair_cnt(a2, 0);
                for (auto &pp : part_pair)
                    for (uint32_t q = 0; q < a2; ++q) pair_cnt[q] += pp[q];
                uint64_t N = 0;  // every token of the context belongs to one of its pairs
                for (uint64_t x : cnt[c]) N += x;
                build_pair_table(pair_cnt, A[c], N / 2, freq[c], rare[c]);
                ntok[c] = A[c];
                tablen[c] = pair_table_len(A[c]);
            } else {
                ntok[c] = build_freqs(cnt[c], freq[c]);
                tablen[c] = ntok[c];
            }
            cum[c].assign(freq[c].size(), 0);
            for (size_t t = 1; t < freq[c].size(); ++t) cum[c][t] = cum[c][t - 1] + freq[c][t - 1];
            tokens += tablen[c];
        }
        const Model model{m, freq, cum, paired, A, rare};
        // tiles, encoded in parallel into per-range buffers
        uint32_t T = tile_count();
        int tchunks = int(std::max<int64_t>(1, std::min<int64_t>(threads, T)));
        std::vector<std::vector<uint8_t>> part_tiles(static_cast<size_t>(tchunks));
        std::vector<std::vector<uint32_t>> part_sizes(static_cast<size_t>(tchunks));
        int64_t tper = (int64_t(T) + tchunks - 1) / tchunks;
        std::vector<char> part_fits(static_cast<size_t>(tchunks), 1);
        parallel_for(tchunks, tchunks, [&](int64_t c0, int64_t c1) {
            std::vector<Event> ev;
            std::vector<uint16_t> words;
            for (int64_t c = c0; c < c1; ++c)
                for (int64_t t = c * tper; t < std::min<int64_t>(T, (c + 1) * tper); ++t) {
                    size_t before = part_tiles[size_t(c)].size();
                    if (!encode_tile(ctx.data(), val.data(), nb, cb, layout, t, K, model, ev, words,
                                     part_tiles[size_t(c)]))
                        part_fits[size_t(c)] = 0;
                    part_sizes[size_t(c)].push_back(uint32_t((part_tiles[size_t(c)].size() - before) / 16));
                }
        });
        for (char f : part_fits)
            if (!f) return {};
        Layout L = layout_for(rows, container, tokens, T);
        size_t tile_bytes = 0;
        for (auto &pt : part_tiles) tile_bytes += pt.size();
        std::vector<uint8_t> out(L.tiles + tile_bytes, 0);
        uint8_t *h = out.data();
        auto put = [](uint8_t *p, uint64_t v, int n) {
            for (int i = 0; i < n; ++i) p[i] = uint8_t(v >> (8 * i));
        };
        write_front(h, L, src.dt, container, rows, cols, T, K, k, m, ntok, tablen, paired, freq, fac.data(),
                    scales.data(), layout);
        uint32_t at = 0;
        size_t d = L.dir, o = L.tiles;
        for (int c = 0; c < tchunks; ++c) {
            for (uint32_t sz : part_sizes[size_t(c)]) {
                put(h + d, at, 4);
                d += 4;
                at += sz;
            }
            std::memcpy(h + o, part_tiles[size_t(c)].data(), part_tiles[size_t(c)].size());
            o += part_tiles[size_t(c)].size();
        }
        put(h + d, at, 4);
        return out;
    }
};

}  // namespace
}  // namespace ep

extern "C" size_t ep_compress_bound(int64_t rows, int64_t cols, const ep_config *cfg) {
    if (rows <= 0 || cols <= 0 || !cfg) return 0;
    double n = double(rows) * double(cols);
    if (cfg->q_index < 0) return size_t(std::floor(cfg->target_bpp * n / 8.0));
    int64_t nb = rows * ((cols + 7) / 8);
    uint32_t K = cfg->blocks_per_lane ? cfg->blocks_per_lane
                                      : (cfg->layout == ep::kLayoutGemm ? 32u
                                                                         : ep::auto_blocks_per_lane(nb, cfg->target_bpp));
    uint64_t T = uint64_t((nb + 32 * int64_t(K) - 1) / (32 * int64_t(K)));
    return ep::layout_for(rows, ep::is_code_container(cfg->container_dtype) ? cfg->container_dtype : 0,
                          7 * ep::kPairMaxTable, T)
               .tiles +
           size_t(T) * (ep::kTileHead + 16) + size_t(5.0 * n);
}

extern "C" int ep_compress_host(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, const ep_config *cfg,
                                void *out, size_t out_cap, size_t *out_nbytes) {
    using namespace ep;
    if (!src || !cfg || !out_nbytes || rows <= 0 || cols <= 0) return EP_ERR_INVALID_ARG;
    *out_nbytes = 0;
    if (!little_endian_host()) return EP_ERR_UNSUPPORTED;
    if (src_dtype != EP_BF16 && src_dtype != EP_FP16 && src_dtype != EP_FP32) return EP_ERR_UNSUPPORTED;
    int container = cfg->container_dtype ? cfg->container_dtype : src_dtype;
    if (container < EP_BF16 || container > EP_FP8_E4M3) return EP_ERR_INVALID_ARG;
    if (cfg->blocks_per_lane > 4096) return EP_ERR_INVALID_ARG;
    if (cfg->coding < EP_CODING_AUTO || cfg->coding > EP_CODING_PAIRED) return EP_ERR_INVALID_ARG;
    if ((rows * ((cols + 7) / 8)) >> 32) return EP_ERR_UNSUPPORTED;
    // the GEMM block order takes whole 128 x 64 operand tiles and 32 blocks per lane
    if (cfg->layout != kLayoutRows && cfg->layout != kLayoutGemm) return EP_ERR_INVALID_ARG;
    if (cfg->layout == kLayoutGemm && !layout_fits(kLayoutGemm, rows, cols, cfg->blocks_per_lane ? cfg->blocks_per_lane : 32u))
        return EP_ERR_INVALID_ARG;

    Encoder E;
    E.src = Source{src, src_dtype};
    E.rows = rows;
    E.cols = cols;
    E.container = container;
    E.coding = cfg->coding;
    E.layout = cfg->layout;
    E.threads = cfg->n_threads > 0 ? cfg->n_threads : int(std::max(1u, std::thread::hardware_concurrency()));
    // finite check
    {
        int64_t n = rows * cols;
        std::vector<char> bad(static_cast<size_t>(E.threads), 0);
        int64_t per = (n + E.threads - 1) / E.threads;
        parallel_for(E.threads, E.threads, [&](int64_t t0, int64_t t1) {
            for (int64_t t = t0; t < t1; ++t)
                for (int64_t i = t * per; i < std::min(n, (t + 1) * per); ++i)
                    if (!std::isfinite(E.src.at(i))) {
                        bad[size_t(t)] = 1;
                        break;
                    }
        });
        for (char b : bad)
            if (b) return EP_ERR_NONFINITE;
    }
    double target = cfg->target_bpp;
    if (!(target >= 0.001) || !(target <= 11.0) || (is_code_container(container) && !(target < 8.0)))
        return EP_ERR_TARGET_RANGE;
    E.prepare();
    E.K = cfg->blocks_per_lane ? cfg->blocks_per_lane
                               : (E.layout == kLayoutGemm ? 32u : auto_blocks_per_lane(E.nb, target));
    int kmax = max_q_index(cols);
    int k;
    if (cfg->q_index >= 0) {
        k = std::min(cfg->q_index, kmax);
    } else {
        double budget = kTargetMargin * target;
        int lo = 0, hi = kmax;
        while (lo < hi) {
            int mid = lo + (hi - lo + 1) / 2;
            if (E.estimate(mid) <= budget)
                lo = mid;
            else
                hi = mid - 1;
        }
        k = lo;
    }
    std::vector<uint8_t> blob;
    for (;;) {
        blob = E.encode(k);
        if (blob.empty()) return EP_ERR_UNSUPPORTED;  // a lane region beyond 65535 words (forced tile size)
        if (cfg->q_index >= 0 || 8.0 * double(blob.size()) <= target * double(rows * cols)) break;
        if (k == 0) {
            *out_nbytes = blob.size();
            return EP_ERR_TARGET_UNREACHABLE;
        }
        --k;
    }
    *out_nbytes = blob.size();
    if (!out || blob.size() > out_cap) return EP_ERR_BUFFER_TOO_SMALL;
    std::memcpy(out, blob.data(), blob.size());
    return EP_OK;
}
