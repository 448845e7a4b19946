// Host-side steps of compression shared by the host compressor (host_encode.cpp) and the device
// compressor (device_encode.cu): the decisions taken from integer histograms (splits, frequency
// tables, the sampled storage estimate) and the bytes in front of the tile section.  Both
// compressors call these same functions, so their streams agree byte for byte.
#pragma once
#include <cstdint>
#include <vector>

#include "format.h"

namespace ep {

// largest resolution index whose lattice coordinates stay below 2^21 for a row of `cols` values
int max_q_index(int64_t cols);

// smallest split allowed for the context with >= 99.9 % of the values below 2^m, from a histogram
// of the values' bit lengths (by_len[0..32])
uint32_t pick_split(const uint64_t *by_len, int ctx);

// frequency table (sum 2^11, every entry below 2^11) from token counts; returns the table length
uint32_t build_freqs(const std::vector<uint64_t> &cnt, std::vector<uint32_t> &f);

// bits per weight estimated from a sample of ns of the nb blocks: the sample's token counts per
// context (at the splits picked on the sample) and its raw extra bits
double estimate_from_counts(const std::vector<uint64_t> *cnt, uint64_t extra_bits, int64_t nb, int64_t ns,
                            int64_t rows, int64_t cols, int container, uint32_t T);

// header, row factors, code scales and frequency tables (everything before the directory);
// `h` holds at least L.dir bytes, zeroed
void write_front(uint8_t *h, const Layout &L, int src_dt, int container, int64_t rows, int64_t cols, uint32_t T,
                 uint32_t K, int k, const uint32_t *m, const uint32_t *ntok, const std::vector<uint32_t> *freq,
                 const float *fac, const float *scales);

bool little_endian_host();

}  // namespace ep
