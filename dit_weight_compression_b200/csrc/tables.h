// tables.h -- pieces both encoders (host threads, GPU) share: symbols, symbol counts, the
// frequency tables built from them (totals 2^prob_bits), the default tile length, the sampled size
// estimate and the blob serialiser.  One definition, so the two encoders cannot drift apart.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <string>
#include <vector>

#include "format.h"

namespace ep {

// Field value -> symbol: f + 127 for |f| <= 127, else the escape symbol.
EP_HD inline int symbol_of(int32_t f) { return (f >= -kAlphabetR && f <= kAlphabetR) ? f + kAlphabetR : kEscape; }

// Symbol counts of the 16 contexts, field j (1..8) given coset c at 8c + j - 1.  Contexts 0 and 8
// (field 1) are the two coset halves of the joint (coset, f1) symbol.
struct Counts {
    std::vector<uint64_t> c = std::vector<uint64_t>(16 * 256, 0);
    uint64_t escapes = 0;
    void add(int coset, const int32_t f[8]) {
        for (int j = 0; j < 8; ++j) {
            int sy = symbol_of(f[j]);
            c[size_t(256 * (8 * coset + j) + sy)]++;
            escapes += sy == kEscape;
        }
    }
    void merge(const Counts& o) {
        for (size_t i = 0; i < c.size(); ++i) c[i] += o.c[i];
        escapes += o.escapes;
    }
};

// Frequencies summing to M from counts: q = max(1, round-half-up(M n / N)) for used symbols, then
// the sum is brought to M -- excess taken one at a time from the largest q (> 1, lowest symbol
// first), deficit given one at a time to the most frequent symbol (lowest symbol first).
inline void quantise_freqs(const uint64_t* n, uint16_t* q, uint32_t M, int nb = 256) {
    uint64_t total = 0;
    for (int s = 0; s < nb; ++s) total += n[s];
    std::fill(q, q + nb, uint16_t(0));
    if (total == 0) return;
    int64_t sum = 0;
    for (int s = 0; s < nb; ++s) {
        if (!n[s]) continue;
        uint64_t v = (2 * uint64_t(M) * n[s] + total) / (2 * total);
        q[s] = uint16_t(std::max<uint64_t>(v, 1));
        sum += q[s];
    }
    while (sum > int64_t(M)) {
        int best = -1;
        for (int s = 0; s < nb; ++s)
            if (q[s] > 1 && (best < 0 || q[s] > q[best])) best = s;
        --q[best];
        --sum;
    }
    while (sum < int64_t(M)) {
        int best = -1;
        for (int s = 0; s < nb; ++s)
            if (n[s] && (best < 0 || n[s] > n[best])) best = s;
        ++q[best];
        ++sum;
    }
}

// The 16 context tables.  Contexts 0 and 8 are quantised together as one 512-symbol table over
// the pairs (coset, f1) (coset-major, so ties go to coset 0 first), the others one by one.  The
// joint symbol (c, s) has frequency q[8c][s] and cumulative frequency joint_cum(c, s): coset 1's
// slots follow all of coset 0's.
struct Tables {
    int prob_bits = kProbBitsDefault;
    uint32_t M = 1u << kProbBitsDefault;
    uint16_t q[16][256];
    uint32_t cum[16][257];
    void build(const Counts& cnt, int pb) {
        prob_bits = pb;
        M = 1u << pb;
        uint64_t nj[512];
        uint16_t qj[512];
        std::copy(&cnt.c[0], &cnt.c[0] + 256, nj);
        std::copy(&cnt.c[256 * 8], &cnt.c[256 * 8] + 256, nj + 256);
        quantise_freqs(nj, qj, M, 512);
        std::copy(qj, qj + 256, q[0]);
        std::copy(qj + 256, qj + 512, q[8]);
        for (int c = 1; c < 16; ++c)
            if (c != 8) quantise_freqs(&cnt.c[size_t(256 * c)], q[c], M);
        for (int c = 0; c < 16; ++c) {
            cum[c][0] = 0;
            for (int s = 0; s < 256; ++s) cum[c][s + 1] = cum[c][s] + q[c][s];
        }
    }
    uint32_t joint_cum(int coset, int s) const { return cum[8 * coset][s] + (coset ? cum[0][256] : 0u); }
    // serialised size of the table section (before padding)
    uint64_t section_bytes() const {
        uint64_t b = 0;
        for (int c = 0; c < 16; ++c) {
            int lo, cnt;
            range(c, lo, cnt);
            b += 4 + 2 * uint64_t(cnt);
        }
        return b;
    }
    void range(int c, int& lo, int& cnt) const {
        int first = -1, last = -1;
        for (int s = 0; s < kEscape; ++s)
            if (q[c][s]) { if (first < 0) first = s; last = s; }
        lo = first < 0 ? 0 : first;
        cnt = first < 0 ? 0 : last - first + 1;
    }
};

// Default tile length: S = clamp(next_pow2(ceil(128 / target)), 16, 1024).
inline int default_steps(double target) {
    double want = std::ceil(128.0 / target);
    int s = 1;
    while (double(s) < want) s *= 2;
    return std::min(1024, std::max(16, s));
}

// Metadata bytes of a blob with these tables: the exact header, table, row-scale, row-maximum and
// tile-offset sections, plus 168 bytes per tile (32 states, 16 region counts, the mean padding).
inline double metadata_bytes(const Tables& T, int64_t rows, int64_t n_tiles) {
    return double(kHeaderBytes + round_up16(T.section_bytes()) + round_up16(4 * uint64_t(rows)) +
                  round_up16(2 * uint64_t(rows)) + round_up16(4 * uint64_t(n_tiles + 1))) +
           double(n_tiles) * (160.0 + 8.0);
}

// Estimated bits per element from the symbol counts of n_sample sampled rows (of `rows`): coded
// bits under the sample's own tables plus 16 bits per escape, scaled to all rows, plus the
// metadata.
inline double estimate_from_counts(const Counts& all, int64_t rows, int64_t cols, int64_t n_sample, int64_t n_tiles,
                                   int prob_bits) {
    Tables T;
    T.build(all, prob_bits);
    double bits = 0.0;
    for (int c = 0; c < 16; ++c)
        for (int sy = 0; sy < 256; ++sy) {
            uint64_t n = all.c[size_t(256 * c + sy)];
            if (n) bits += double(n) * -std::log2(double(T.q[c][sy]) / double(T.M));
        }
    double payload = (double(rows) / double(n_sample)) * (bits / 8.0 + 2.0 * double(all.escapes));
    return 8.0 * (metadata_bytes(T, rows, n_tiles) + payload) / (double(rows) * double(cols));
}

// Write the blob: header, table section, row scales, row maxima, tile offsets (from the tile byte
// sizes) and room for the stream.  The stream's bytes are left zero; its offset is returned in
// *off_stream.  Returns false (with `why`) when the stream would exceed the tile-offset range.
bool assemble_blob(int dtype, int64_t rows, int64_t cols, int S, double s, const Tables& T,
                   const std::vector<float>& alpha, const std::vector<uint16_t>& rowmax,
                   const std::vector<uint64_t>& tile_bytes, std::vector<uint8_t>& blob, uint64_t* off_stream,
                   std::string& why);

}  // namespace ep
