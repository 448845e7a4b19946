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

// frequency table (sum `scale`, every entry below it) from counts; returns the table length
uint32_t build_freqs(const std::vector<uint64_t> &cnt, std::vector<uint32_t> &f, uint32_t scale = kProbScale);

// last token seen, plus one
uint32_t seen_len(const std::vector<uint64_t> &cnt);

// whether a stream pairs coordinates 1..6 (coding: EP_CODING_*; m: the splits; cnt1, cnt2: the
// token counts of contexts 1 and 2)
bool pair_eligible(int coding, int64_t nb, const uint32_t *m, const std::vector<uint64_t> &cnt1,
                   const std::vector<uint64_t> &cnt2);

// pair table of a context with alphabet length A from the counts of its token pairs inside the
// base (B * B of them, B = pair_base(A)) and of all its pairs (N): pairs outside the base and rare
// pairs go to the escape symbol B * B, then the table is normalised to 2^12; `rare` flags the
// escaped pair indices inside the base
void build_pair_table(std::vector<uint64_t> pair_cnt, uint32_t A, uint64_t N, std::vector<uint32_t> &f,
                      std::vector<uint8_t> &rare);

// bits per weight estimated from a sample of ns of the nb blocks: the sample's token counts per
// context (at the splits m picked on the sample) and its raw extra bits
double estimate_from_counts(const std::vector<uint64_t> *cnt, const uint32_t *m, int coding, uint64_t extra_bits,
                            int64_t nb, int64_t ns, int64_t rows, int64_t cols, int container, uint32_t T);

// header, row factors, code scales and frequency tables (everything before the directory);
// `h` holds at least L.dir bytes, zeroed.  ntok: the header's per-context lengths; tablen: the
// entries of freq[c] written (the pair tables' A * A + 1 for a paired stream's contexts 1, 2)
void write_front(uint8_t *h, const Layout &L, int src_dt, int container, int64_t rows, int64_t cols, uint32_t T,
                 uint32_t K, int k, const uint32_t *m, const uint32_t *ntok, const uint32_t *tablen, bool paired,
                 const std::vector<uint32_t> *freq, const float *fac, const float *scales, int layout);

bool little_endian_host();

}  // namespace ep
