// decode_launch.h -- what the host side of the decode (decode.cu) and the kernel units
// (decode_unit.cu, one per output container and table layout) share: the kernel parameter
// blocks, the shared-memory geometry of every table layout and CTA width, the rule that picks
// them for a launch, the status bits, and one table of launch functions per unit.
//
// The kernels are templates over the output container and the table layout; each pair's
// instantiations live in a translation unit of their own, so the library builds in parallel.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "format.h"

namespace ep {
namespace dec {

constexpr uint32_t kWaitSpins = 1u << 22;                     // bounded mbarrier wait (~0.3 s)
// Decode tables: [0] the joint (coset, f1) symbol; [1 + 7c + (j - 2)] field j = 2..8 given coset c.
constexpr int kDecodeTables = 15;
// 10-bit totals: one packed u32 entry per slot, 1024 slots per table (4 KB), 60 KB in all.
// 12-bit totals: a u8 symbol per slot, 4096 slots per table (4 KB), then a 4-byte entry per
// symbol -- 512 for the joint table, 256 for each other -- 60 KB + 16 KB.
constexpr uint32_t kCtxBytes = 4096;                          // one table's slot block, either total
constexpr uint32_t kSlotBytes = kDecodeTables * kCtxBytes;    // 61440
// The per-symbol entries of coset 1 start kCosetSkew bytes past a whole number of rows, so that a
// warp whose lanes read the same symbol of the same field in both cosets hits different banks.
constexpr uint32_t kCosetSkew = 64;
constexpr uint32_t kSymEntryBytes = 16 * 256 * 4 + kCosetSkew;  // 16448 (12-bit totals only)
// 12-bit totals, hybrid layouts 11, 15, 13 and 14: the joint table and the next kND fields (none
// for layout 11; f2 for layout 15; f2, f3 for layout 13; f2, f3, f4 for layout 14) given each
// coset as direct words, one u32 per slot (16 KB a table); the other 7 - kND fields given each
// coset as symbol bytes (4 KB a table) and 4-byte per-symbol entries (1 KB a table).  Layout 11
// takes 86 KB, 15 108 KB, 13 130 KB, 14 152 KB.
constexpr uint32_t kHDirect = 4 * 4096;                       // one direct table: 16384
template <int LAY>
struct Hybrid {
    static constexpr uint32_t kND = LAY == 14 ? 3 : LAY == 13 ? 2 : LAY == 15 ? 1 : 0;  // direct fields per coset after the joint table
    static constexpr uint32_t kNB = 7 - kND;                   // two-lookup fields per coset
    static constexpr uint32_t kL1 = (1 + 2 * kND) * kHDirect;  // their symbol bytes (16384 / 81920 / 114688)
    static constexpr uint32_t kL2 = kL1 + 2 * kNB * kCtxBytes; // their 4-byte entries
    static constexpr uint32_t kBytes = kL2 + 2 * kNB * 1024 + kCosetSkew;  // 88128 / 110656 / 133184 / 155712
};
__host__ __device__ constexpr bool is_hybrid(int lay) { return lay == 11 || lay == 13 || lay == 14 || lay == 15; }

// Table layouts: 10 = 10-bit totals, one packed word per slot; 12 = 12-bit totals, two lookups
// per symbol; 11, 13, 14 and 15 = 12-bit totals, hybrid.
template <int LAY>
struct TableGeo {
    static_assert(LAY >= 10 && LAY <= 15, "table layouts are 10 to 15");
    static constexpr uint32_t kBytes =
        LAY == 10 ? kSlotBytes : LAY == 12 ? kSlotBytes + kSymEntryBytes : Hybrid<LAY>::kBytes;
    static constexpr uint32_t kPiece = kBytes / 4;             // bytes per table bulk copy
    static_assert(kPiece % 16 == 0, "bulk copies move multiples of 16 bytes");
};
inline uint32_t table_bytes(int lay) {
    return lay == 10 ? TableGeo<10>::kBytes
         : lay == 11 ? TableGeo<11>::kBytes
         : lay == 12 ? TableGeo<12>::kBytes
         : lay == 13 ? TableGeo<13>::kBytes
         : lay == 14 ? TableGeo<14>::kBytes : TableGeo<15>::kBytes;
}

// kOutE4M3Row: the FP8 container with a per-row scale -- an E4M3 payload normalised per row to
// the format's range, plus one fp32 scale per row.
enum OutKind { kOutBF16 = 0, kOutFP16 = 1, kOutE4M3 = 2, kOutF32 = 3, kOutFields = 4, kOutI8 = 5, kOutE4M3Row = 6 };

// Status word bits (sticky, cleared by ep_decode_status).
enum : uint32_t {
    kStOverrun = 1u,   // a lane read past its region, the regions overrun the tile, or a tile's
                       // extent lies outside the stream
    kStState = 2u,     // a lane did not end in state 2^16
    kStLeftover = 4u,  // a region's two lanes did not meet, or 16+ bytes follow the regions
    kStTimeout = 8u    // a bulk-copy wait hit its limit
};

// What the decode of one blob needs (small: a grouped launch passes up to kMaxGroup of them as
// its kernel parameter).
struct Params {
    const uint8_t* tables;      // expanded decode tables (TableGeo::kBytes), or null: expand in-kernel
    const uint32_t* tile_off;   // n_tiles + 1 offsets, 16-byte units
    const uint8_t* stream;      // stream section
    const float* alpha;         // per-row fp32 scales
    const uint16_t* rowmax;     // per-row largest |2 y| (row-scaled FP8 only)
    float* sigma;               // per-row scale output (row-scaled FP8 only)
    void* out;
    uint32_t* status;
    int64_t rows, cols, row_stride, n_vectors;
    uint64_t stream_bytes;      // size of the stream section: every tile must lie inside it
    uint32_t vec_per_row;       // < 2^31 (checked when the blob is parsed)
    uint32_t steps, n_tiles;
    uint32_t joint_split;       // slots of coset 0 in the joint (coset, f1) table
};

// Where the blob keeps the compact frequency tables the decode table is expanded from.
struct TableSrc {
    const uint8_t* blob;        // device copy of the serialised blob
    uint32_t q_off[kFieldContexts];
    uint32_t esc_q[kFieldContexts];
    uint32_t lo[kFieldContexts];
    uint32_t n[kFieldContexts];
};

// Run-time controls of a single-blob launch.
struct Ctl {
    uint32_t wait_spins = kWaitSpins;  // iterations of a bounded mbarrier wait before it gives up
    uint32_t probe_tx = 0;             // test only: > 0 makes the table wait expect this many
                                       // bytes that no copy delivers, so the wait must give up
};

// A set of blobs in one launch: blob m owns CTAs [cta0, cta0 + ncta).
constexpr int kMaxGroup = 28;
struct GroupEntry {
    Params p;
    uint32_t cta0, ncta;
    uint32_t vec, esc;
};
struct GroupParams {
    uint32_t n;
    GroupEntry e[kMaxGroup];
};
static_assert(sizeof(GroupParams) <= 4000, "a group must fit the classic 4 KB kernel parameter space");

// ---- shared-memory geometry ------------------------------------------------------------------
constexpr uint32_t kSmemOptin = 232448;  // 227 KB: the largest dynamic shared memory of one CTA
constexpr uint32_t kAlignSlack = 4096;    // the table starts on a 4 KB boundary of the shared window
constexpr uint32_t kBufSlack = 80;        // bytes after a tile buffer that two steps may over-read

// CTA widths: 16, 20, 24 or 32 warps, each warp with a tile buffer of Geo<WARPS, LAY>::kBuf bytes:
//   layout 10: 10336, 8240, 6848, 5120;  layout 11: 8656, 6912, 5744, 4288;
//   layout 12: 9296, 7424, 6176, 4608;   layout 15: 7248, 5792, 4800, 3584;
//   layout 13: 5840, 4656;  layout 14: 4432
// (layout 13 leaves room for 16 or 20 warps, layout 14 for 16).  A tile larger than its warp's
// buffer is read from global memory.
constexpr int kWarpsNarrow = 16, kWarps20 = 20, kWarpsMid = 24, kWarpsWide = 32;

// Per-warp tile buffer size for a CTA of WARPS warps: what the 227 KB leave after the tables.
template <int WARPS, int LAY>
struct Geo {
    static constexpr uint32_t kBuf =
        ((kSmemOptin - kAlignSlack - TableGeo<LAY>::kBytes - 64 - WARPS * (kBufSlack + 8) - 16) / WARPS) & ~15u;
};
template <int WARPS, int LAY>
struct Smem {
    alignas(16) uint8_t tab[TableGeo<LAY>::kBytes];                      // decode tables
    alignas(16) uint8_t tbuf[WARPS][Geo<WARPS, LAY>::kBuf + kBufSlack];  // one staged tile per warp
    unsigned long long bar[WARPS];                                      // tile staging, one per warp
    unsigned long long tbar;                                            // the table's bulk copies
    unsigned long long pbar;                                            // the wait-limit probe
};
using Smem32x10 = Smem<32, 10>;
using Smem32x12 = Smem<32, 12>;
static_assert(offsetof(Smem32x10, tbuf) == TableGeo<10>::kBytes && offsetof(Smem32x12, tbuf) == TableGeo<12>::kBytes,
              "table block must be contiguous");
template <int WARPS, int LAY>
constexpr bool fits_smem() { return sizeof(Smem<WARPS, LAY>) + kAlignSlack <= kSmemOptin; }
static_assert(fits_smem<16, 10>() && fits_smem<20, 10>() && fits_smem<24, 10>() && fits_smem<32, 10>() &&
              fits_smem<16, 12>() && fits_smem<20, 12>() && fits_smem<24, 12>() && fits_smem<32, 12>() &&
              fits_smem<16, 13>() && fits_smem<20, 13>() && fits_smem<16, 14>() && fits_smem<16, 11>() &&
              fits_smem<20, 11>() && fits_smem<24, 11>() && fits_smem<32, 11>() && fits_smem<16, 15>() &&
              fits_smem<20, 15>() && fits_smem<24, 15>() && fits_smem<32, 15>(),
              "shared memory budget");
inline bool width_ok(int warps, int lay) {
    if (lay == 14) return warps == kWarpsNarrow;
    return warps == kWarpsNarrow || warps == kWarps20 || (lay != 13 && (warps == kWarpsMid || warps == kWarpsWide));
}
inline uint32_t tile_buffer_bytes(int warps, int lay) {
    switch (lay * 100 + warps) {
        case 1016: return Geo<16, 10>::kBuf;
        case 1020: return Geo<20, 10>::kBuf;
        case 1024: return Geo<24, 10>::kBuf;
        case 1032: return Geo<32, 10>::kBuf;
        case 1116: return Geo<16, 11>::kBuf;
        case 1120: return Geo<20, 11>::kBuf;
        case 1124: return Geo<24, 11>::kBuf;
        case 1132: return Geo<32, 11>::kBuf;
        case 1216: return Geo<16, 12>::kBuf;
        case 1220: return Geo<20, 12>::kBuf;
        case 1224: return Geo<24, 12>::kBuf;
        case 1232: return Geo<32, 12>::kBuf;
        case 1316: return Geo<16, 13>::kBuf;
        case 1320: return Geo<20, 13>::kBuf;
        case 1416: return Geo<16, 14>::kBuf;
        case 1516: return Geo<16, 15>::kBuf;
        case 1520: return Geo<20, 15>::kBuf;
        case 1524: return Geo<24, 15>::kBuf;
        case 1532: return Geo<32, 15>::kBuf;
        default: return 0;
    }
}
// Index of a layout's expanded tables in a device copy of a blob.
inline int layout_index(int lay) {
    return lay == 10 ? 0 : lay == 12 ? 1 : lay == 13 ? 2 : lay == 14 ? 3 : lay == 11 ? 4 : 5;
}
constexpr int kLayouts = 6;

// ---- launch shape: table layout and CTA width ------------------------------------------------
// A launch of n_tiles tiles over `ctas` CTAs (one per SM) runs in rounds: each warp decodes its
// tiles one after another, so the time is about the number of rounds, ceil(n_tiles / (warps *
// ctas)), times one tile's rANS chain, stretched by the warps that share the SM.  The chain of a
// vector is 8 one-load symbols (layout 10), 4 one-load + 4 two-load (14), 3 + 5 (13), 2 + 6 (15),
// 1 + 7 (11) or 8 two-load (12): weights 8, 12, 13, 14, 15, 16 at ~45 cycles a one-load symbol.  Each warp past 16 adds
// 1/64 (fitted to the measured choices between 16-, 24- and 32-warp CTAs).  A shape is usable when
// its tile buffers hold the largest tile.  The cheapest usable shape wins; on a tie, the layout
// with the shorter chain, then the narrower width when a single round suffices (more registers
// per thread, no idle warps), else the wider (more chains per SM).
struct LaunchShape {
    int lay, warps;
};
inline uint32_t chain_weight(int lay) {
    return lay == 10 ? 8u : lay == 14 ? 12u : lay == 13 ? 13u : lay == 15 ? 14u : lay == 11 ? 15u : 16u;
}
inline uint64_t shape_cost(int lay, int warps, uint64_t n_tiles, uint64_t ctas) {
    const uint64_t slots = uint64_t(warps) * (ctas ? ctas : 1);
    return ((n_tiles + slots - 1) / slots) * chain_weight(lay) * uint64_t(48 + warps);
}
inline bool shape_better(LaunchShape a, LaunchShape b, uint64_t n_tiles, uint64_t ctas) {
    const uint64_t ca = shape_cost(a.lay, a.warps, n_tiles, ctas), cb = shape_cost(b.lay, b.warps, n_tiles, ctas);
    if (ca != cb) return ca < cb;
    if (a.lay != b.lay) return chain_weight(a.lay) < chain_weight(b.lay);
    const bool one_round = n_tiles <= uint64_t(a.warps) * ctas && n_tiles <= uint64_t(b.warps) * ctas;
    return one_round ? a.warps < b.warps : a.warps > b.warps;
}
// The CTA width for tables already fixed to layout `lay`.
inline int cta_warps(int lay, uint64_t max_tile_bytes, uint64_t n_tiles, uint64_t ctas) {
    LaunchShape best{lay, 0};
    for (int w : {kWarpsNarrow, kWarps20, kWarpsMid, kWarpsWide}) {
        if (!width_ok(w, lay) || max_tile_bytes > tile_buffer_bytes(w, lay)) continue;
        if (!best.warps || shape_better(LaunchShape{lay, w}, best, n_tiles, ctas)) best.warps = w;
    }
    return best.warps ? best.warps : kWarpsNarrow;  // no buffer holds the largest tile: read it from global memory
}
// Layout and width of a launch for blobs with 2^prob_bits frequency totals.  `wide_ok` false (a
// launch that runs 16-warp CTAs only) considers 16 warps alone, and every layout but 14.  When no buffer holds the largest
// tile: layout 10, or layout 13 if its 16-warp buffers do, else 12, in 16-warp CTAs (the
// oversized tiles are read from global memory).
inline LaunchShape launch_shape(int prob_bits, uint64_t max_tile_bytes, uint64_t n_tiles, uint64_t ctas, bool wide_ok) {
    LaunchShape best{0, 0};
    const int lays12[5] = {14, 13, 15, 11, 12}, lays10[1] = {10};
    const int* lays = prob_bits == 10 ? lays10 : lays12;
    const int nl = prob_bits == 10 ? 1 : 5;
    for (int k = 0; k < nl; ++k)
        for (int w : {kWarpsNarrow, kWarps20, kWarpsMid, kWarpsWide}) {
            if (!width_ok(w, lays[k]) || (!wide_ok && (w != kWarpsNarrow || lays[k] == 14))) continue;
            if (max_tile_bytes > tile_buffer_bytes(w, lays[k])) continue;
            const LaunchShape s{lays[k], w};
            if (!best.warps || shape_better(s, best, n_tiles, ctas)) best = s;
        }
    if (best.warps) return best;
    if (prob_bits == 10) return LaunchShape{10, kWarpsNarrow};
    return LaunchShape{max_tile_bytes <= Geo<16, 13>::kBuf ? 13 : 12, kWarpsNarrow};
}
inline int table_layout(int prob_bits, uint64_t max_tile_bytes, uint64_t n_tiles, uint64_t ctas, bool wide_ok) {
    return launch_shape(prob_bits, max_tile_bytes, n_tiles, ctas, wide_ok).lay;
}

// ---- launch functions, one table per output container and table layout ----------------------
struct LaunchCtx {
    int device;  // CUDA ordinal (current device)
    int sms;     // its SM count
};

// The launches of one output container with one table layout; each (container, layout) pair is
// compiled in a unit of its own (decode_unit.cu).  The CTA width is in warps: 16, 20, 24 or 32 for
// layouts 10, 11, 12 and 15, 16 or 20 for layout 13, 16 for layout 14.  A null entry does not exist: the
// fields test hook and the row-scaled FP8 container have single-blob launches only, and the
// allocation-free launch takes every layout but 14.
struct Launchers {
    // one blob; `dependent`: launch as a programmatic dependent of the previous decode
    int (*single)(const Params& p, bool vec, int warps, bool esc, const Ctl& ctl, cudaStream_t st, const LaunchCtx& c,
                  bool dependent);
    // a set of blobs over `grid` CTAs
    int (*group)(const GroupParams& g, uint32_t grid, int warps, cudaStream_t st, const LaunchCtx& c);
    // one blob, tables expanded in every CTA, status in caller-provided memory; never allocates
    int (*noalloc)(const Params& p, const TableSrc& ts, bool vec, bool esc, cudaStream_t st, const LaunchCtx& c);
};

// kLaunch_<container>_<layout>, one per unit.
#define EP_DECLARE_UNITS(o) \
    extern const Launchers kLaunch_##o##_10, kLaunch_##o##_12, kLaunch_##o##_13, kLaunch_##o##_14, kLaunch_##o##_11, \
        kLaunch_##o##_15;
EP_DECLARE_UNITS(0)
EP_DECLARE_UNITS(1)
EP_DECLARE_UNITS(2)
EP_DECLARE_UNITS(3)
EP_DECLARE_UNITS(4)
EP_DECLARE_UNITS(5)
EP_DECLARE_UNITS(6)
#undef EP_DECLARE_UNITS
static_assert(kOutBF16 == 0 && kOutFP16 == 1 && kOutE4M3 == 2 && kOutF32 == 3 && kOutFields == 4 && kOutI8 == 5 &&
              kOutE4M3Row == 6, "unit names use the container numbers");

inline const Launchers* unit_launchers(int out_kind, int lay) {
#define EP_UNIT_ROW(o) \
    {&kLaunch_##o##_10, &kLaunch_##o##_12, &kLaunch_##o##_13, &kLaunch_##o##_14, &kLaunch_##o##_11, &kLaunch_##o##_15}
    static const Launchers* const table[7][kLayouts] = {EP_UNIT_ROW(0), EP_UNIT_ROW(1), EP_UNIT_ROW(2), EP_UNIT_ROW(3),
                                                        EP_UNIT_ROW(4), EP_UNIT_ROW(5), EP_UNIT_ROW(6)};
#undef EP_UNIT_ROW
    if (out_kind < 0 || out_kind > 6 || lay < 10 || lay > 15) return nullptr;
    return table[out_kind][layout_index(lay)];
}

}  // namespace dec
}  // namespace ep
