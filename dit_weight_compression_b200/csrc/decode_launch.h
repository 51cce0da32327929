// decode_launch.h -- what the host side of the decode (decode.cu) and the per-container kernel
// units (decode_<container>.cu) share: the kernel parameter blocks, the shared-memory geometry,
// the status bits, and one table of launch functions per output container.
//
// The kernels are templates over the output container; each container's instantiations live in
// a translation unit of their own (decode_bf16.cu, ...), so the library builds in parallel.
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
// 12-bit totals, hybrid: the joint table and f2, f3 given each coset as direct words, one u32 per
// slot (5 tables of 16 KB), the other 10 tables as symbol bytes (4 KB each) and 4-byte entries
// (1 KB each) -- 130 KB, which leaves 16-warp CTAs 5.8 KB tile buffers.
constexpr uint32_t kHDirect = 4 * 4096;                       // one direct table: 16384
constexpr uint32_t kHL1 = 5 * kHDirect;                       // 81920: symbol bytes of f4..f8
constexpr uint32_t kHL2 = kHL1 + 10 * kCtxBytes;              // 122880: their 4-byte entries
constexpr uint32_t kHybridBytes = kHL2 + 10 * 1024 + kCosetSkew;  // 133184

// Table layouts: 10 = 10-bit totals, one packed word per slot; 12 = 12-bit totals, two lookups
// per symbol; 13 = 12-bit totals, hybrid (16-warp CTAs only).
template <int LAY>
struct TableGeo {
    static_assert(LAY == 10 || LAY == 12 || LAY == 13, "table layouts are 10, 12 and 13");
    static constexpr uint32_t kBytes = LAY == 10 ? kSlotBytes : LAY == 12 ? kSlotBytes + kSymEntryBytes : kHybridBytes;
    static constexpr uint32_t kPiece = kBytes / 4;             // bytes per table bulk copy
};
inline uint32_t table_bytes(int lay) {
    return lay == 10 ? TableGeo<10>::kBytes : lay == 12 ? TableGeo<12>::kBytes : TableGeo<13>::kBytes;
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

// CTA widths: 32, 24 or 16 warps, each warp with a tile buffer of Geo<WARPS, LAY>::kBuf bytes
// (5120, 6848 or 10336 with layout 10; 4608, 6176 or 9296 with layout 12; 5840 with layout 13,
// which leaves room for 16 warps only); a tile larger than its warp's buffer is read from global
// memory.
constexpr int kWarpsWide = 32, kWarpsMid = 24, kWarpsNarrow = 16;

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
static_assert(sizeof(Smem<32, 10>) + kAlignSlack <= kSmemOptin && sizeof(Smem<24, 10>) + kAlignSlack <= kSmemOptin &&
              sizeof(Smem<16, 10>) + kAlignSlack <= kSmemOptin && sizeof(Smem<32, 12>) + kAlignSlack <= kSmemOptin &&
              sizeof(Smem<24, 12>) + kAlignSlack <= kSmemOptin && sizeof(Smem<16, 12>) + kAlignSlack <= kSmemOptin &&
              sizeof(Smem<16, 13>) + kAlignSlack <= kSmemOptin,
              "shared memory budget");
inline uint32_t tile_buffer_bytes(int warps, int lay) {
    if (lay == 10) return warps == 32 ? Geo<32, 10>::kBuf : warps == 24 ? Geo<24, 10>::kBuf : Geo<16, 10>::kBuf;
    if (lay == 12) return warps == 32 ? Geo<32, 12>::kBuf : warps == 24 ? Geo<24, 12>::kBuf : Geo<16, 12>::kBuf;
    return Geo<16, 13>::kBuf;
}
// Index of a layout's expanded tables in a device copy of a blob.
inline int layout_index(int lay) { return lay == 10 ? 0 : lay == 12 ? 1 : 2; }
constexpr int kLayouts = 3;

// The layout a launch of n_tiles tiles (largest max_tile_bytes) decodes with on a device of `sms`
// SMs.  10-bit totals take layout 10.  12-bit totals take layout 12 in 24- or 32-warp CTAs when
// there are more tiles than 16-warp CTAs hold at once and every tile fits the 24-warp buffers
// (more independent rANS chains per SM are worth the second lookup of three more symbols per
// vector); else the hybrid when every tile fits its 16-warp buffers; else layout 12.  `wide_ok`
// false (a launch that runs 16-warp CTAs only) skips the first rule.
inline int table_layout(int prob_bits, uint64_t max_tile_bytes, uint64_t n_tiles, int sms, bool wide_ok) {
    if (prob_bits == 10) return 10;
    if (wide_ok && n_tiles > uint64_t(kWarpsNarrow) * uint64_t(sms > 0 ? sms : 0) &&
        max_tile_bytes <= Geo<kWarpsMid, 12>::kBuf)
        return 12;
    return max_tile_bytes <= Geo<16, 13>::kBuf ? 13 : 12;
}
// The CTA width of such a launch over `ctas` CTAs: 16 warps when they hold every tile at once (the
// 16-warp kernel has the most registers per thread); else the widest whose buffers hold the
// largest tile (more chains per SM, fewer rounds of tiles); layout 13 runs 16 warps only.
inline int cta_warps(int lay, uint64_t max_tile_bytes, uint64_t n_tiles, uint64_t ctas) {
    if (lay == 13 || n_tiles <= uint64_t(kWarpsNarrow) * ctas) return kWarpsNarrow;
    if (max_tile_bytes <= tile_buffer_bytes(kWarpsWide, lay)) return kWarpsWide;
    if (max_tile_bytes <= tile_buffer_bytes(kWarpsMid, lay)) return kWarpsMid;
    return kWarpsNarrow;
}

// ---- launch functions, one table per output container ----------------------------------------
struct LaunchCtx {
    int device;  // CUDA ordinal (current device)
    int sms;     // its SM count
};

// Every function takes the table layout lay (10, 12 or 13) and the CTA width in warps (16, 24 or
// 32; layout 13 runs 16).
struct Launchers {
    // one blob; `dependent`: launch as a programmatic dependent of the previous decode
    int (*single)(const Params& p, int lay, bool vec, int warps, bool esc, const Ctl& ctl, cudaStream_t st,
                  const LaunchCtx& c, bool dependent);
    // a set of blobs, all with the same layout, over `grid` CTAs
    int (*group)(const GroupParams& g, int lay, uint32_t grid, int warps, cudaStream_t st, const LaunchCtx& c);
    // one blob, tables expanded in every CTA, status in caller-provided memory; never allocates
    int (*noalloc)(const Params& p, const TableSrc& ts, int lay, bool vec, bool esc, cudaStream_t st,
                   const LaunchCtx& c);
};

extern const Launchers kLaunchBF16, kLaunchFP16, kLaunchE4M3, kLaunchF32, kLaunchI8, kLaunchFields, kLaunchE4M3Row;

}  // namespace dec
}  // namespace ep
