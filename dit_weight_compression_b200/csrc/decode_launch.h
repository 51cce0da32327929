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
constexpr uint32_t kCtxBytes = 4 * kProbTotal;                // one context's packed table: 4 KB
// Decode tables: [0] the joint (coset, f1) symbol; [1 + 7c + (j - 2)] field j = 2..8 given coset c.
constexpr int kDecodeTables = 15;
constexpr uint32_t kTableBytes = kDecodeTables * kCtxBytes;   // 61440
constexpr uint32_t kTablePiece = kTableBytes / 4;             // bytes per table bulk copy (15 KB)

enum OutKind { kOutBF16 = 0, kOutFP16 = 1, kOutE4M3 = 2, kOutF32 = 3, kOutFields = 4, kOutI8 = 5 };

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
    const uint8_t* tables;      // expanded decode table (kTableBytes), or null: expand in-kernel
    const uint32_t* tile_off;   // n_tiles + 1 offsets, 16-byte units
    const uint8_t* stream;      // stream section
    const float* alpha;         // per-row fp32 scales
    void* out;
    uint32_t* status;
    int64_t rows, cols, row_stride, n_vectors;
    uint64_t stream_bytes;      // size of the stream section: every tile must lie inside it
    uint32_t vec_per_row;       // < 2^31 (checked when the blob is parsed)
    uint32_t steps, n_tiles;
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
constexpr int kMaxGroup = 32;
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

// CTA widths: 32 warps with 4992-byte tile buffers, or 16 warps with 10080-byte buffers; a tile
// larger than its warp's buffer is read from global memory.
constexpr int kWarpsWide = 32, kWarpsNarrow = 16;

// Per-warp tile buffer size for a CTA of WARPS warps: what the 227 KB leave after the table.
template <int WARPS>
struct Geo {
    static constexpr uint32_t kBuf =
        ((kSmemOptin - kAlignSlack - kTableBytes - 64 - WARPS * (kBufSlack + 8) - 16) / WARPS) & ~15u;
};

template <int WARPS>
struct Smem {
    uint32_t tab[kDecodeTables][kProbTotal];                        // packed decode tables, 60 KB
    alignas(16) uint8_t tbuf[WARPS][Geo<WARPS>::kBuf + kBufSlack];  // one staged tile per warp
    unsigned long long bar[WARPS];                                  // tile staging, one per warp
    unsigned long long tbar;                                        // the table's bulk copies
    unsigned long long pbar;                                        // the wait-limit probe
};
static_assert(offsetof(Smem<32>, tbuf) == kTableBytes, "table block must be contiguous");
static_assert(sizeof(Smem<32>) + kAlignSlack <= kSmemOptin && sizeof(Smem<16>) + kAlignSlack <= kSmemOptin,
              "shared memory budget");

// ---- launch functions, one table per output container ----------------------------------------
struct LaunchCtx {
    int device;  // CUDA ordinal (current device)
    int sms;     // its SM count
};

struct Launchers {
    // one blob; `dependent`: launch as a programmatic dependent of the previous decode
    int (*single)(const Params& p, bool vec, bool wide, bool esc, const Ctl& ctl, cudaStream_t st,
                  const LaunchCtx& c, bool dependent);
    // a set of blobs over `grid` CTAs
    int (*group)(const GroupParams& g, uint32_t grid, bool wide, cudaStream_t st, const LaunchCtx& c);
    // one blob, tables expanded in every CTA, status in caller-provided memory; never allocates
    int (*noalloc)(const Params& p, const TableSrc& ts, bool vec, bool esc, cudaStream_t st, const LaunchCtx& c);
};

extern const Launchers kLaunchBF16, kLaunchFP16, kLaunchE4M3, kLaunchF32, kLaunchI8, kLaunchFields;

}  // namespace dec
}  // namespace ep
