// format.h -- internal description of the compressed blob shared by the host encoder, the blob
// validator and the GPU launch code of the library.
//
// The blob holds what "EntroPack lattice compression" (documentation page, section "Encoding
// and reconstruction") says must travel with the rANS-coded fields: the frequency tables, one
// scale per row, and the per-tile bookkeeping.  Byte layout (little-endian, every section 16-byte aligned):
//
//   header, 96 bytes:  "EPK1" | u16 version = 4 | u8 dtype | u8 R = 127 | u64 rows | u64 cols |
//                      u32 S | u32 n_tiles | f64 s | u64 total bytes | u64 table offset |
//                      u64 row-scale offset | u64 tile-offset offset | u64 stream offset |
//                      u64 row-maximum offset | u8 prob_bits | 7 zero bytes
//   tables:            for c = 0, 1 and j = 1..8: u16 q(escape), u8 lo, u8 n,
//                      u16 q[lo .. lo + n - 1]; the two j = 1 tables are the coset halves of
//                      one table over the pairs (coset, f1), summing to M together
//   row scales:        f32 per row
//   row maxima:        u16 per row, the row's largest |2 y| over its real columns
//   tile offsets:      u32[n_tiles + 1], in 16-byte units from the stream start
//   stream:            per tile: 32 u32 initial rANS states (lane order), 16 u16 region word
//                      counts, the regions (lane 2p's words forward from the region start, lane
//                      2p+1's backward from its end), zero padding to a multiple of 16 bytes
//
// Symbols: field value f with |f| <= 127 is the symbol f + 127; any other value is the escape
// symbol 255 followed by the raw int16 word.  A vector is 8 rANS symbols: (coset, f1), then
// f2..f8 given the coset.  Frequencies of every used context sum to M = 2^prob_bits: 4096
// (12-bit totals, the format's fixed choice and the default) or 1024 (10-bit, an option).
#pragma once

#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

// Functions the device code of the library shares with its host code.
#ifdef __CUDACC__
#define EP_HD __host__ __device__
#else
#define EP_HD
#endif

namespace ep {

constexpr uint32_t kVersion = 4;
constexpr int kAlphabetR = 127;
constexpr int kEscape = 255;
constexpr int kProbBitsDefault = 12;              // M = 4096; 10 (M = 1024) is the other choice
EP_HD inline bool prob_bits_ok(int pb) { return pb == 10 || pb == 12; }
constexpr uint32_t kStateLow = 1u << 16;          // rANS lower bound, 16-bit renormalisation
constexpr int kLanes = 32;                        // interleaved states per tile
constexpr int kPairs = kLanes / 2;                // lanes 2p, 2p+1 share word region p
constexpr int kFieldContexts = 16;                // (coset c, field j) -> 8c + j - 1; 0 and 8
                                                  // together: the joint (coset, f1) table
constexpr size_t kHeaderBytes = 96;
constexpr size_t kTileHeadBytes = 4 * kLanes + 2 * kPairs;  // 32 u32 states + 16 u16 counts
constexpr double kTargetMin = 0.001, kTargetMax = 11.0;

enum Dtype : int { kBF16 = 1, kFP16 = 2, kE4M3 = 3, kF32 = 4, kI8 = 5 };

inline int dtype_bytes(int dt) {
    switch (dt) {
        case kBF16: case kFP16: return 2;
        case kE4M3: case kI8: return 1;
        case kF32: return 4;
        default: return 0;
    }
}

EP_HD inline uint64_t round_up16(uint64_t n) { return (n + 15) & ~uint64_t(15); }

// Parsed, validated header of a blob plus the decoded frequency tables.
struct BlobLayout {
    int dtype = 0;
    int prob_bits = 0;            // frequency totals M = 2^prob_bits
    int64_t rows = 0, cols = 0, vec_per_row = 0, n_vectors = 0;
    uint32_t steps = 0, n_tiles = 0;
    uint64_t max_tile_bytes = 0;  // largest tile (selects the decoder's shared-memory layout)
    int has_escape = 0;           // some field context gives the escape symbol a frequency
    double scale = 0.0;
    uint64_t total = 0, off_tables = 0, off_alpha = 0, off_rowmax = 0, off_offsets = 0, off_stream = 0;
    uint32_t joint_split = 0;     // slots of coset 0 in the joint (coset, f1) table
    // field contexts: escape frequency, symbol range, byte offset of q[] inside the blob
    uint16_t esc_q[kFieldContexts] = {};
    uint8_t lo[kFieldContexts] = {}, n[kFieldContexts] = {};
    uint32_t q_offset[kFieldContexts] = {};
};

// Little-endian readers / writers.
inline uint16_t rd16(const uint8_t* p) { return uint16_t(p[0] | (p[1] << 8)); }
inline uint32_t rd32(const uint8_t* p) {
    return uint32_t(p[0]) | (uint32_t(p[1]) << 8) | (uint32_t(p[2]) << 16) | (uint32_t(p[3]) << 24);
}
inline uint64_t rd64(const uint8_t* p) { return uint64_t(rd32(p)) | (uint64_t(rd32(p + 4)) << 32); }
inline void wr16(uint8_t* p, uint32_t v) { p[0] = uint8_t(v); p[1] = uint8_t(v >> 8); }
inline void wr32(uint8_t* p, uint32_t v) { wr16(p, v & 0xFFFF); wr16(p + 2, v >> 16); }
inline void wr64(uint8_t* p, uint64_t v) { wr32(p, uint32_t(v)); wr32(p + 4, uint32_t(v >> 32)); }

// Validate serialised bytes; on failure returns false and sets `why`.
bool parse_blob(const uint8_t* data, size_t n, BlobLayout& L, std::string& why);

// Host encoder input: a rows x cols matrix of container bit patterns in host memory.
struct EncodeInput {
    const void* bits;
    int dtype;
    int64_t rows, cols, row_stride;
};
struct EncodeOptions {
    int steps_per_tile = 0;  // S; 0 = default rule
    int threads = 0;         // 0 = all hardware threads
    double scale = 0.0;      // > 0: skip the scale search
    bool rd_refine = false;  // per-row rate-distortion refinement
    int prob_bits = kProbBitsDefault;  // frequency totals 2^prob_bits (12 or 10)
};
// Returns 0, -3 (shape/size limits) or -4 (non-finite input); `why` explains a failure.
int encode(const EncodeInput& in, double target, const EncodeOptions& opt, std::vector<uint8_t>& blob,
           std::string& why);
// The same encoder with its parallel work on the GPU, for a device tensor (in.bits on the current
// device); the same bytes.  Also -6 (a CUDA call failed) and -7 (device memory).  No refinement.
int encode_gpu(const EncodeInput& in, double target, const EncodeOptions& opt, std::vector<uint8_t>& blob,
               std::string& why);

}  // namespace ep
