// decode_device.cuh -- the fused GPU decompression kernel for sm_100a, and its launch functions.
//
// "EntroPack lattice compression" (documentation page, section "Encoding and reconstruction"):
// a single fused GPU operation takes the coded fields back to lattice points, scales each row and
// returns a tensor with the original shape and element type.  Per the arXiv abstract every tile
// decodes on its own, which is what lets the GPU work on all of them at once.
//
// One kernel does the whole path.  Work split:
//   * one warp per tile; the tile's 32 interleaved rANS states live one per lane;
//   * one persistent CTA per SM (16, 20, 24 or 32 warps, with the table layout chosen per launch
//     by launch_shape in decode_launch.h; grid = min(#SM, #tiles)); tile t goes to CTA t mod grid,
//     so every SM gets an equal share even when there are few tiles;
//   * decode tables, for the joint (coset, f1) symbol and for f2..f8 given each coset (15
//     tables).  With 10-bit totals: one packed 32-bit entry per slot of the 1024-slot range,
//     {slot - cum(s), s (2 s for f8), escape flag, coset bit, q(s)} -- 60 KB -- so one
//     shared-memory load per symbol gives everything the state update needs.  With 12-bit totals
//     the per-slot entries would take 240 KB, more than an SM has, so most symbols take two
//     loads: the slot's symbol byte (4096 per table, 60 KB), then that symbol's packed
//     {q(s), 4096 - cum(s)} word (16 KB).  Layouts 13 and 14 give the joint table and the next 2
//     or 3 fields one packed word per slot instead, as far as shared memory allows.  Either way
//     the state update is a shift-add and an extraction side by side, then one multiply-add.
//     The tables are expanded once per blob, device and layout by a small kernel into
//     a block next to the device copy; every CTA stages that block into shared memory with bulk
//     copies, overlapped with the fetch of its first tiles.  (The allocation-free entry point
//     expands them inside each CTA instead.);
//   * words: every lane reads its own word stream.  Lanes 2p and 2p+1 share region p of the tile
//     (one forward from the region start, one backward from its end); a warp-shuffle prefix sum
//     over the 16 region counts gives every lane its start.  The whole tile is staged into a
//     per-warp shared-memory buffer by one bulk copy (the next tile is prefetched into L2); each
//     lane has its next word loaded before it needs it, so a renormalisation costs a compare and
//     a predicated multiply-add on the dependent chain;
//   * per step a lane decodes one 8-vector: 8 rANS symbols, (coset, f1) then f2..f8 (each
//     followed by its conditional refill), then the raw words of its escaped fields; fields are
//     inverted in registers (z8 = 2 f8 + parity, y = z + c/2), multiplied by the row's fp32 scale,
//     converted one pair per cvt and written as one 16-byte store per lane (a 512-byte contiguous
//     run per warp for BF16/FP16).  Steps are software-pipelined: step k + 1's symbols are decoded
//     before step k is written, so the writes fill the stalls of the rANS chain.
// No tensor cores: the path is table lookups and integer arithmetic, bound by HBM bytes and by
// the latency and issue slots of that arithmetic, not by a contraction.
//
// Every (output container, table layout) pair instantiates these templates in a translation unit
// of its own (decode_unit.cu, compiled once per pair), which exports one Launchers table.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <mutex>
#include <string>
#include <type_traits>

#include "blob.h"
#include "decode_launch.h"

namespace ep {
namespace dec {
namespace {

constexpr uint32_t kFull = 0xFFFFFFFFu;

// Packed decode-table entry of slot u, symbol s = the one with cum(s) <= u < cum(s) + q(s) (for
// the joint table the symbol is the pair (c, s) and cum runs over coset 0's symbols first):
//   bits  0..9   u - cum(s)           (< q(s) <= 1024)
//   bits 10..18  s at bit 10 for fields 1..7 (bit 18 zero), s at bit 11 for field 8 (bit 10 zero)
//   bit  19      s is the escape symbol
//   bit  20      the coset c          (joint table only)
//   bits 21..31  q(s)                 (<= 1024)
// so the state update x <- q (x >> 10) + u - cum(s) takes two field extractions, and one mask
// puts s (or 2 s for field 8, whose lattice coordinate is 2 f8 + parity) in place as mantissa
// bits of the float the reconstruction starts from.
constexpr uint32_t kEntryBiasMask = 0x3FFu;
constexpr uint32_t kEntrySymShift = 10;
constexpr uint32_t kEntryEsc = 1u << 19;
constexpr uint32_t kEntryCosetShift = 20;
constexpr uint32_t kEntryQShift = 21;
constexpr uint32_t kSlots10 = 1024;

// 12-bit totals.  Symbol byte of slot u of table t at [4096 t + u] (for the joint table the f1
// symbol of the slot's coset half; the coset is u >= the coset-0 total).  Per-symbol entry of
// field j (1: the joint table, its coset-1 cumulative frequencies following all of coset 0's)
// given coset c at [kSlotBytes + c (8 * 1024 + kCosetSkew) + 1024 (j - 1) + 4 s]:
//   bits  0..12  q(s)                 (<= 4096; the whole entry is 0 for a symbol the table does not hold)
//   bits 19..31  4096 - cum(s)        (1..4096; the joint table's coset-1 symbols follow coset 0's)
// With the slot u = x mod 4096 and u' = x | 0xFFFFF000 (= u - 4096 mod 2^32, formed next to the
// slot's address), the state update is x <- q (x >> 12) + (u' + (entry >> 19)), mod 2^32 equal to
// q (x >> 12) + u - cum(s): one shift-add and one extraction after the load, then the multiply-add.
constexpr uint32_t kE12QMask = 0x1FFFu;
constexpr uint32_t kE12NegCumShift = 19;
__device__ __forceinline__ uint32_t pack_entry12(uint32_t q, uint32_t cum) {
    return q ? q | ((4096u - cum) << kE12NegCumShift) : 0u;
}

// Shared addresses of the decode tables a step reads.
template <int LAY>
struct Tab {
    uint32_t t;        // 10-bit: the packed entries, 4 KB aligned
};
template <>
struct Tab<12> {
    uint32_t s1;       // symbol bytes, 4 KB aligned
    uint32_t e2;       // per-symbol entries
    uint32_t s1split;  // s1 + the slots of coset 0 in the joint table
};
// Layouts 11, 15, 13 and 14 (12-bit totals, hybrid with D = Hybrid<LAY>::kND direct fields per coset and
// B = 7 - D two-lookup ones), at `base` (4 KB aligned): the joint table's direct words at base;
// field j = 2 .. D + 1 given coset c at base + kHDirect (1 + D c + j - 2); symbol bytes of field
// j = D + 2 .. 8 given c at base + kL1 + 4096 (B c + j - D - 2); their 4-byte entries (as in
// layout 12) at base + kL2 + c (B * 1024 + kCosetSkew) + 1024 (j - D - 2).  A direct word of slot
// u holding s:
//   bits  0..11  q(s) - 1
//   bits 12..19  s
//   bits 20..31  u - cum(s)
// so x <- (q - 1) (x >> 12) + ((x >> 12) + (word >> 20)): the shift-add and the extraction of
// q - 1 run side by side after the load.
struct TabHybrid {
    uint32_t base;
    uint32_t split;    // slots of coset 0 in the joint table
};
template <>
struct Tab<11> : TabHybrid {};
template <>
struct Tab<15> : TabHybrid {};
template <>
struct Tab<13> : TabHybrid {};
template <>
struct Tab<14> : TabHybrid {};
__device__ __forceinline__ uint32_t pack_direct(uint32_t off, uint32_t s, uint32_t q) {
    return q ? (q - 1) | (s << 12) | (off << 20) : 0u;
}

// Scratch of the table expansion: frequencies and cumulative frequencies of every context.
struct BuildScratch {
    uint16_t q[kFieldContexts][256];
    uint16_t cum[kFieldContexts][257];
};
static_assert(sizeof(BuildScratch) <= 16 * Geo<32, 12>::kBuf, "expansion scratch fits the tile buffers");

// ---- PTX wrappers ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(unsigned long long* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// 1-D bulk copy global -> this CTA's own shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, unsigned long long* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ bool mbar_test(unsigned long long* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded, warp-uniform wait for the phase of `bar` with the given parity.
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, uint32_t parity, uint32_t limit = kWaitSpins) {
    for (uint32_t it = 0; it < limit; ++it) {
        if (__all_sync(kFull, mbar_test(bar, parity))) return true;
        if (it >= 16) __nanosleep(64);
    }
    return false;
}

// Shared-memory loads at 32-bit shared-window addresses (plus a constant byte offset).
template <int OFF = 0>
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF));
    return v;
}
// Shared address of slot (x mod M) of a 4 KB-aligned table at `base`: a mask and a multiply-add,
// which keeps one of the two steps off the integer ALU pipe.
__device__ __forceinline__ uint32_t slot_addr(uint32_t x, uint32_t base) {
    uint32_t a;
    asm("{\n .reg .b32 t;\n and.b32 t, %1, 1023;\n mad.lo.u32 %0, t, 4, %2;\n}" : "=r"(a) : "r"(x), "r"(base));
    return a;
}

// Prefetch `bytes` (a multiple of 16) at a 16-byte aligned global address into L2.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// A lane's word stream, read from the warp's shared-memory copy of the tile.  `wp` is the
// shared address of the lane's next word and `wn` that word, loaded right after the previous
// one was used -- well before it is needed, so a refill costs a compare and a multiply-add on
// the dependent chain.  Predicated loads keep the warp converged.
struct SmemReader {
    uint32_t wp, wn;
    int32_t wd;  // +2 (lane 2p, forward) or -2 (lane 2p+1, backward)
    __device__ __forceinline__ void consume_if(bool take) {
        asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %2, 0;\n @p add.u32 %1, %1, %3;\n @p ld.shared.u16 %0, [%1];\n}"
                     : "+r"(wn), "+r"(wp)
                     : "r"(uint32_t(take)), "r"(wd));
    }
    // words consumed since `wp` was `wp0`
    __device__ __forceinline__ uint32_t consumed(uint32_t wp0) const { return uint32_t(int32_t(wp - wp0) / wd); }
};

// The same for a tile too large for the buffer: words come from global memory, every address
// clamped into the tile.
struct GlobalReader {
    const uint8_t* tile;
    int32_t off, hi, wd;  // byte offset of the next word; last legal word offset; +-2
    uint32_t wn;
    __device__ __forceinline__ void consume_if(bool take) {
        off += take ? wd : 0;
        const uint8_t* src = tile + min(max(off, 0), hi);
        asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %1, 0;\n @p ld.global.nc.u16 %0, [%2];\n}"
                     : "+r"(wn)
                     : "r"(uint32_t(take)), "l"(src));
    }
    __device__ __forceinline__ uint32_t consumed(int32_t off0) const { return uint32_t((off - off0) / wd); }
};

// Renormalisation after one decoded symbol: a lane whose state fell below 2^16 shifts in its
// next word (x * 2^16 + w) and loads the word after it.
template <class Reader>
__device__ __forceinline__ void renorm(uint32_t& x, Reader& rd, bool active) {
    const bool need = active && x < kStateLow;
    x = need ? __byte_perm(rd.wn, x, 0x5410) : x;
    rd.consume_if(need);
}
// The same for full steps from shared memory, as one predicated block: compare, multiply-add
// (on the FMA pipe, which the rest of the step leaves idle), advance, load -- no materialised
// predicate or select.
__device__ __forceinline__ void renorm(uint32_t& x, SmemReader& rd) {
    asm volatile(
        "{\n .reg .pred p;\n setp.lt.u32 p, %0, 65536;\n @p mad.lo.u32 %0, %0, 65536, %1;\n"
        " @p add.u32 %2, %2, %3;\n @p ld.shared.u16 %1, [%2];\n}"
        : "+r"(x), "+r"(rd.wn), "+r"(rd.wp)
        : "r"(rd.wd));
}
template <bool FULL, class Reader>
__device__ __forceinline__ void renorm_step(uint32_t& x, Reader& rd, bool active) {
    if constexpr (FULL && std::is_same<Reader, SmemReader>::value) renorm(x, rd);
    else renorm(x, rd, active);
}

// ---- table expansion -------------------------------------------------------------------------
// Largest symbol s with cum[s] <= slot: the symbol of that slot (its frequency is not zero).
__device__ __forceinline__ uint32_t slot_symbol(const uint16_t* cum, uint32_t slot) {
    uint32_t s = 0;
#pragma unroll
    for (uint32_t step = 128; step; step >>= 1)
        if (cum[s + step] <= slot) s += step;
    return s;
}

__device__ __forceinline__ uint32_t pack_entry(uint32_t bias, uint32_t s, uint32_t q, uint32_t coset, uint32_t sh) {
    return bias | (s << sh) | (s == uint32_t(kEscape) ? kEntryEsc : 0u) |
           (coset << kEntryCosetShift) | (q << kEntryQShift);
}

// Layout 11, 15, 13 or 14 from the per-context frequencies and cumulative frequencies in `scr`: the
// 1 + 2D direct tables, the 2B symbol-byte tables, then the 4-byte entries of those 2B.
template <int WARPS, int LAY>
__device__ void build_hybrid(uint8_t* tab, const BuildScratch& scr) {
    constexpr uint32_t D = Hybrid<LAY>::kND, B = Hybrid<LAY>::kNB;
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int P = WARPS >= 15 ? WARPS / 15 : 1;
    constexpr uint32_t kSlotsPerPart = 4096u / P;
    const uint32_t split = scr.cum[0][256];
    uint32_t* dir = reinterpret_cast<uint32_t*>(tab);
    for (uint32_t item = warp; item < uint32_t(15 * P); item += WARPS) {
        const uint32_t ti = item / P, part = item % P;
        if (ti == 0) {  // the joint table, direct: coset 0's slots, then coset 1's
            for (uint32_t w = lane; w < kSlotsPerPart; w += 32) {
                const uint32_t slot = part * kSlotsPerPart + w;
                const uint32_t c = slot < split ? 0u : 1u;
                const uint32_t local = slot - (c ? split : 0u);
                const uint16_t* cum = scr.cum[8 * c];
                const uint32_t sy = slot_symbol(cum, local);
                dir[slot] = pack_direct(local - cum[sy], sy, scr.q[8 * c][sy]);
            }
            continue;
        }
        // ti 1..2D: f2..f(D+1) given c (direct); ti 2D+1..14: f(D+2)..f8 given c (symbol bytes)
        const bool direct = ti <= 2 * D;
        const uint32_t k = direct ? ti - 1 : ti - 1 - 2 * D;
        constexpr uint32_t Dd = D ? D : 1;  // layout 11 has no direct field after the joint table
        const uint32_t c = direct ? k / Dd : k / B;
        const uint32_t j = direct ? 2 + k % Dd : 2 + D + k % B;
        const uint32_t ctx = 8 * c + j - 1;
        const uint16_t* cum = scr.cum[ctx];
        const uint16_t* qs = scr.q[ctx];
        uint32_t* dst32 = direct ? dir + ti * 4096u : nullptr;
        uint8_t* dst8 = direct ? nullptr : tab + Hybrid<LAY>::kL1 + k * kCtxBytes;
        if (cum[256] != 4096u) {  // context never used by this blob (the host checked the rest)
            for (uint32_t w = lane; w < kSlotsPerPart; w += 32) {
                if (direct) dst32[part * kSlotsPerPart + w] = 0;
                else dst8[part * kSlotsPerPart + w] = 0;
            }
            continue;
        }
        const uint32_t first = part * kSlotsPerPart + lane;
        uint32_t sy = slot_symbol(cum, first);
        uint32_t c0 = cum[sy], next = cum[sy + 1];
        for (uint32_t w = lane; w < kSlotsPerPart; w += 32) {
            const uint32_t slot = part * kSlotsPerPart + w;
            while (next <= slot) {
                ++sy;
                c0 = next;
                next = cum[sy + 1];
            }
            if (direct) dst32[slot] = pack_direct(slot - c0, sy, qs[sy]);
            else dst8[slot] = uint8_t(sy);
        }
    }
    for (uint32_t i = threadIdx.x; i < 2 * B * 256; i += WARPS * 32) {
        const uint32_t row = i >> 8, sy = i & 255;        // row = B c + j - D - 2
        const uint32_t c = row / B, ctx = 8 * c + 1 + D + row % B;
        const uint32_t q = scr.q[ctx][sy];
        uint32_t* ent = reinterpret_cast<uint32_t*>(tab + Hybrid<LAY>::kL2 + c * kCosetSkew + 1024 * row);
        ent[sy] = pack_entry12(q, uint32_t(scr.cum[ctx][sy]));
    }
}

// Fills the decode tables at `tab` (shared memory, TableGeo<LAY>::kBytes) from the blob's compact
// frequency tables (16 contexts; 0 and 8 together are the joint (coset, f1) table).  `scr` is
// shared-memory scratch (BuildScratch) that the caller does not use meanwhile.
template <int WARPS, int LAY>
__device__ void build_tables(uint8_t* tab, BuildScratch& scr, const TableSrc& p) {
    constexpr uint32_t M = LAY == 10 ? 1024u : 4096u;
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // (a) per context: frequencies of symbols 8*lane .. 8*lane+7 and their cumulative sums
    for (uint32_t ctx = warp; ctx < kFieldContexts; ctx += WARPS) {
        const uint32_t lo = p.lo[ctx], n = p.n[ctx];
        const uint16_t* qa = reinterpret_cast<const uint16_t*>(p.blob + p.q_off[ctx]);
        uint32_t q[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t s = 8 * lane + i, v = 0;
            if (s == kEscape) v = p.esc_q[ctx];
            else if (s >= lo && s < lo + n) v = __ldg(qa + (s - lo));
            q[i] = v;
            sum += v;
        }
        uint32_t inc = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t t = __shfl_up_sync(kFull, inc, o);
            if (lane >= uint32_t(o)) inc += t;
        }
        uint32_t c = inc - sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            scr.q[ctx][8 * lane + i] = uint16_t(q[i]);
            scr.cum[ctx][8 * lane + i] = uint16_t(c);  // <= M for a valid table
            c += q[i];
        }
        if (lane == 31) scr.cum[ctx][256] = uint16_t(min(c, 0xFFFFu));
    }
    __syncthreads();
    if constexpr (is_hybrid(LAY)) {
        build_hybrid<WARPS, LAY>(tab, scr);
        return;
    }
    // (b) slot -> entry (10-bit: the packed word; 12-bit: the symbol byte).  Lane l of a warp
    // writes slots it*32 + l of its part (one contiguous run per store instruction); each lane
    // walks its symbol forward as its slots grow.
    constexpr int P = WARPS >= 15 ? WARPS / 15 : 1;
    constexpr uint32_t kSlotsPerPart = M / P;
    static_assert(M % P == 0, "parts split the slots evenly");
    uint32_t* tab32 = reinterpret_cast<uint32_t*>(tab);
    auto put = [&](uint32_t ti, uint32_t slot, uint32_t bias, uint32_t sy, uint32_t q, uint32_t coset, uint32_t sh) {
        if constexpr (LAY == 10) tab32[ti * kSlots10 + slot] = pack_entry(bias, sy, q, coset, sh);
        else tab[ti * kCtxBytes + slot] = uint8_t(sy);
    };
    for (uint32_t item = warp; item < uint32_t(kDecodeTables * P); item += WARPS) {
        const uint32_t ti = item / P, part = item % P;
        if (ti == 0) {  // the joint table: coset 0's slots, then coset 1's
            const uint32_t split = scr.cum[0][256];
            for (uint32_t w = lane; w < kSlotsPerPart; w += 32) {
                const uint32_t slot = part * kSlotsPerPart + w;
                const uint32_t c = slot < split ? 0u : 1u;
                const uint32_t local = slot - (c ? split : 0u);
                const uint16_t* cum = scr.cum[8 * c];
                const uint32_t sy = slot_symbol(cum, local);
                put(0, slot, local - cum[sy], sy, scr.q[8 * c][sy], c, kEntrySymShift);
            }
            continue;
        }
        const uint32_t ctx = 8 * ((ti - 1) / 7) + 1 + (ti - 1) % 7;  // field j = 2..8 given coset c
        const uint16_t* cum = scr.cum[ctx];
        const uint16_t* qs = scr.q[ctx];
        const uint32_t sh = (ti - 1) % 7 == 6 ? kEntrySymShift + 1 : kEntrySymShift;  // field 8: 2 s
        if (cum[256] != M) {  // context never used by this blob (the host checked the rest)
            for (uint32_t w = lane; w < kSlotsPerPart; w += 32) put(ti, part * kSlotsPerPart + w, 0, 0, 0, 0, 0);
            continue;
        }
        const uint32_t first = part * kSlotsPerPart + lane;
        uint32_t sy = slot_symbol(cum, first);
        uint32_t c0 = cum[sy], next = cum[sy + 1];
        for (uint32_t w = lane; w < kSlotsPerPart; w += 32) {
            const uint32_t slot = part * kSlotsPerPart + w;
            while (next <= slot) {
                ++sy;
                c0 = next;
                next = cum[sy + 1];
            }
            put(ti, slot, slot - c0, sy, qs[sy], 0u, sh);
        }
    }
    if constexpr (LAY == 12) {
        // (c) the per-symbol entries of field j (1..8) given coset c (the joint table's coset-1
        // cumulative frequencies follow coset 0's; a field's carry its table's offset in the block)
        const uint32_t split = scr.cum[0][256];
        for (uint32_t i = threadIdx.x; i < 16 * 256; i += WARPS * 32) {
            const uint32_t c = i >> 11, j = 1 + ((i >> 8) & 7), sy = i & 255;
            const uint32_t ctx = 8 * c + j - 1;
            const uint32_t q = scr.q[ctx][sy];
            const uint32_t cum = scr.cum[ctx][sy] + (j == 1 && c ? split : 0u);
            uint32_t* ent = reinterpret_cast<uint32_t*>(tab + kSlotBytes + c * (8 * 1024 + kCosetSkew) + 1024 * (j - 1));
            ent[sy] = pack_entry12(q, cum);
        }
    }
}

// ---- output conversion -----------------------------------------------------------------------
template <int OUT>
struct OutElem {
    static constexpr int kBytes = (OUT == kOutE4M3 || OUT == kOutE4M3Row || OUT == kOutI8) ? 1 : (OUT == kOutF32 ? 4 : 2);
};

// Eight values to eight consecutive elements at `dst` (aligned to the vector's size).
template <int OUT>
__device__ __forceinline__ void store_vec(uint8_t* dst, const float v[8]) {
    if constexpr (OUT == kOutBF16) {
        uint4 u;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]), h3 = __floats2bfloat162_rn(v[6], v[7]);
        u.x = *reinterpret_cast<uint32_t*>(&h0);
        u.y = *reinterpret_cast<uint32_t*>(&h1);
        u.z = *reinterpret_cast<uint32_t*>(&h2);
        u.w = *reinterpret_cast<uint32_t*>(&h3);
        __stcs(reinterpret_cast<uint4*>(dst), u);
    } else if constexpr (OUT == kOutFP16) {
        uint4 u;
        __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
        __half2 h2 = __floats2half2_rn(v[4], v[5]), h3 = __floats2half2_rn(v[6], v[7]);
        u.x = *reinterpret_cast<uint32_t*>(&h0);
        u.y = *reinterpret_cast<uint32_t*>(&h1);
        u.z = *reinterpret_cast<uint32_t*>(&h2);
        u.w = *reinterpret_cast<uint32_t*>(&h3);
        __stcs(reinterpret_cast<uint4*>(dst), u);
    } else if constexpr (OUT == kOutI8) {
        // nearest integer, ties to even, saturated to [-128, 127]; bytes packed in order
        int32_t q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = max(-128, min(127, __float2int_rn(v[i])));
        const uint32_t lo = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
        const uint32_t hi = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
        __stcs(reinterpret_cast<uint2*>(dst), make_uint2(lo, hi));
    } else if constexpr (OUT == kOutE4M3 || OUT == kOutE4M3Row) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = __nv_cvt_float2_to_fp8x2(make_float2(v[2 * i], v[2 * i + 1]), __NV_SATFINITE, __NV_E4M3);
        __stcs(reinterpret_cast<uint2*>(dst), make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16)));
    } else {
        float4* o = reinterpret_cast<float4*>(dst);
        __stcs(o, make_float4(v[0], v[1], v[2], v[3]));
        __stcs(o + 1, make_float4(v[4], v[5], v[6], v[7]));
    }
}

template <int OUT>
__device__ __forceinline__ void store_one(uint8_t* dst, float v) {
    if constexpr (OUT == kOutBF16) *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(v);
    else if constexpr (OUT == kOutFP16) *reinterpret_cast<__half*>(dst) = __float2half_rn(v);
    else if constexpr (OUT == kOutE4M3 || OUT == kOutE4M3Row)
        *dst = uint8_t(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
    else if constexpr (OUT == kOutI8) *dst = uint8_t(max(-128, min(127, __float2int_rn(v))));
    else *reinterpret_cast<float*>(dst) = v;
}

// ---- the row factor a step multiplies the lattice coordinates by -------------------------------
// The FP8 container with a per-row scale ("EntroPack: ... at Arbitrary Bitrates", abstract: FP8 is
// one of the containers, and the stored rate is set apart from the restored precision): row r's
// payload is E4M3(RNE_fp32(y * g_r)), g_r = RNE_fp32(896 / m_r) with alpha_r's sign (0 for an
// all-zero row or alpha_r = 0), m_r the row's largest |2 y|, so the row's largest value meets 448;
// sigma_r = RNE_fp32(|alpha_r| m_r / 896) restores it.  Every other container multiplies by alpha_r.
__device__ __forceinline__ float row_gain(float a, uint32_t m2) {
    const float g = __fdiv_rn(896.0f, float(m2));  // correctly rounded
    return (m2 == 0 || a == 0.0f) ? 0.0f : (a < 0.0f ? -g : g);
}
// (the double quotient of these operands is never a float rounding tie unless the exact value is,
// so rounding it to float is the correct rounding of |alpha| m / 896)
__device__ __forceinline__ float row_sigma(float a, uint32_t m2) {
    return __double2float_rn(__ddiv_rn(double(fabsf(a)) * double(m2), 896.0));
}
template <int OUT>
__device__ __forceinline__ float row_factor(const Params& p, int64_t row) {
    const float a = __ldg(p.alpha + row);
    if constexpr (OUT == kOutE4M3Row) return row_gain(a, __ldg(p.rowmax + row));
    else return a;
}

// ---- one step: every lane decodes (at most) one 8-vector --------------------------------------
// Where a lane's current vector goes: vector kcol of row `row`, whose first element is at optr,
// and that row's scale.
struct Pos {
    uint8_t* optr;
    int64_t row;
    uint32_t kcol;
    float a;
};

template <int OUT>
__device__ __forceinline__ Pos first_pos(const Params& p, int64_t v) {
    Pos s;
    if constexpr (OUT == kOutFields) {
        s.optr = static_cast<uint8_t*>(p.out) + 18 * v;  // 9 int16 per vector
        s.row = 0;
        s.kcol = 0;
        s.a = 0.0f;
    } else {
        s.row = v / p.vec_per_row;
        s.kcol = uint32_t(v - s.row * p.vec_per_row);
        s.optr = static_cast<uint8_t*>(p.out) + (s.row * p.row_stride + 8 * int64_t(s.kcol)) * OutElem<OUT>::kBytes;
        s.a = v < p.n_vectors ? row_factor<OUT>(p, s.row) : 0.0f;
    }
    return s;
}

// The lane's next vector is 32 further on; the row scale is reloaded only when the row changes.
// WIDE: rows hold at least 32 vectors, so a step crosses at most one row end (no branch).
template <int OUT, bool WIDE>
__device__ __forceinline__ void advance(const Params& p, Pos& s) {
    if constexpr (OUT == kOutFields) {
        s.optr += 32 * 18;
    } else {
        constexpr int es = OutElem<OUT>::kBytes;
        const int64_t wrap = (p.row_stride - 8 * int64_t(p.vec_per_row)) * es;
        s.kcol += 32;
        s.optr += 32 * 8 * es;
        if constexpr (WIDE) {
            const bool w = s.kcol >= p.vec_per_row;
            s.kcol -= w ? p.vec_per_row : 0u;
            s.row += w ? 1 : 0;
            s.optr += w ? wrap : 0;
            if (w && s.row < p.rows) s.a = row_factor<OUT>(p, s.row);
        } else if (s.kcol >= p.vec_per_row) {
            do {
                s.kcol -= p.vec_per_row;
                ++s.row;
                s.optr += wrap;
            } while (s.kcol >= p.vec_per_row);
            s.a = s.row < p.rows ? row_factor<OUT>(p, s.row) : 0.0f;
        }
    }
}

// How a lane's output position moves from step to step.
//   kWalkRows32: rows hold a multiple of 32 vectors (and every vector is one aligned store), so the
//                32 lanes of a warp change rows at the same step: the steps of a tile run row by
//                row, with nothing but the output pointer moving inside a row;
//   kWalkWide:   rows of at least 32 vectors: a step crosses at most one row end;
//   kWalkNarrow: shorter rows.
enum Walk { kWalkRows32 = 0, kWalkWide = 1, kWalkNarrow = 2 };

// The decoded symbols of one step, held between the rANS chain and the writes so that a step's
// reconstruction can overlap the next step's chain.
struct StepSyms {
    uint32_t e[8];
    int32_t f[8];  // only for the escape path and the fields output
    uint32_t c;
    bool from_symbols;
};

// ESC: the blob's tables give the escape symbol a frequency, so a field may be a raw word.
template <bool ESC, bool FULL, class Reader>
__device__ __forceinline__ void step_symbols10(uint32_t tab, Reader& rd, uint32_t& x, bool active, StepSyms& s) {
    if (FULL) active = true;
    // (coset, f1) as one symbol of the joint table, then f2..f8 from the 7 tables of that coset.
    // A lane past the last vector still loads (from its masked slot, inside the table) but keeps x.
    uint32_t* e = s.e;
    uint32_t acc = 0;
    e[0] = lds_u32<0>(slot_addr(x, tab));
    if (active) x = (e[0] >> kEntryQShift) * (x >> 10) + (e[0] & kEntryBiasMask);
    renorm_step<FULL>(x, rd, active);
    if (ESC) acc = e[0];
    const uint32_t c = (e[0] >> kEntryCosetShift) & 1u;
    s.c = c;
    const uint32_t tb = tab + kCtxBytes + c * (7u * kCtxBytes);  // 4 KB aligned
#define EP_FIELD(j)                                                                    \
    {                                                                                  \
        const uint32_t ent = lds_u32<((j) - 1) * kCtxBytes>(slot_addr(x, tb)); \
        if (active) x = (ent >> kEntryQShift) * (x >> 10) + (ent & kEntryBiasMask); \
        renorm_step<FULL>(x, rd, active);                                              \
        e[j] = ent;                                                                    \
        if (ESC) acc |= ent;                                                           \
    }
    EP_FIELD(1) EP_FIELD(2) EP_FIELD(3) EP_FIELD(4) EP_FIELD(5) EP_FIELD(6) EP_FIELD(7)
#undef EP_FIELD

    s.from_symbols = true;
    if constexpr (ESC) {  // defined on both paths (an undefined join costs the kernel its registers)
#pragma unroll
        for (int j = 0; j < 8; ++j) s.f[j] = 0;
    }
    if (ESC && __any_sync(kFull, active && (acc & kEntryEsc))) {
        // escaped fields: the lane's raw words after its renormalisation words, by field
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const bool mine = active && (e[j] & kEntryEsc);
            s.f[j] = mine ? int32_t(int16_t(rd.wn)) : int32_t((e[j] >> (kEntrySymShift + (j == 7))) & 255u) - kAlphabetR;
            rd.consume_if(mine);
        }
        s.from_symbols = false;
    }
}

// The same with 12-bit totals: per symbol the slot's symbol byte, then that symbol's entry.
// s.e[j] holds the symbol s_j itself.
template <bool ESC, bool FULL, class Reader>
__device__ __forceinline__ void step_symbols12(const Tab<12>& T, Reader& rd, uint32_t& x, bool active, StepSyms& s) {
    if (FULL) active = true;
    uint32_t* e = s.e;
    uint32_t acc = 0;                          // largest symbol: the escape symbol is the largest
    // (coset, f1): the slot's half of the joint table gives the coset (known before the loads
    // return), its byte the f1 symbol.  A lane past the last vector still loads but keeps x.
    uint32_t c;
    {
        const uint32_t a1 = (x & 4095u) | T.s1, um = x | 0xFFFFF000u;
        c = a1 >= T.s1split ? 1u : 0u;
        const uint32_t sy = lds_u8<0>(a1);
        const uint32_t en = lds_u32<0>(T.e2 + (8u * 1024u + kCosetSkew) * c + 4u * sy);
        if (active) x = (en & kE12QMask) * (x >> 12) + (um + (en >> kE12NegCumShift));
        renorm_step<FULL>(x, rd, active);
        e[0] = sy;
        if (ESC) acc = sy;
    }
    s.c = c;
    const uint32_t b1 = T.s1 + kCtxBytes + c * (7u * kCtxBytes);        // field 2's symbol bytes given c
    const uint32_t b2 = T.e2 + 1024u + c * (8u * 1024u + kCosetSkew);   // field 2's entries given c
#define EP_FIELD12(j)                                                                         \
    {                                                                                         \
        const uint32_t um = x | 0xFFFFF000u;                                                  \
        const uint32_t sy = lds_u8<((j) - 1) * kCtxBytes>((x & 4095u) | b1);                  \
        const uint32_t en = lds_u32<((j) - 1) * 1024>(b2 + 4u * sy);                          \
        if (active) x = (en & kE12QMask) * (x >> 12) + (um + (en >> kE12NegCumShift));        \
        renorm_step<FULL>(x, rd, active);                                                     \
        e[j] = sy;                                                                            \
        if (ESC) acc = max(acc, sy);                                                          \
    }
    EP_FIELD12(1) EP_FIELD12(2) EP_FIELD12(3) EP_FIELD12(4) EP_FIELD12(5) EP_FIELD12(6) EP_FIELD12(7)
#undef EP_FIELD12

    s.from_symbols = true;
    if constexpr (ESC) {
#pragma unroll
        for (int j = 0; j < 8; ++j) s.f[j] = 0;
    }
    if (ESC && __any_sync(kFull, active && acc == uint32_t(kEscape))) {
        // escaped fields: the lane's raw words after its renormalisation words, by field
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const bool mine = active && e[j] == uint32_t(kEscape);
            s.f[j] = mine ? int32_t(int16_t(rd.wn)) : int32_t(e[j]) - kAlphabetR;
            rd.consume_if(mine);
        }
        s.from_symbols = false;
    }
}

// Layouts 11, 15, 13 and 14: (coset, f1) and the next D fields from direct words (one load each), the
// rest as in layout 12.
template <int LAY, bool ESC, bool FULL, class Reader>
__device__ __forceinline__ void step_symbols_hybrid(const Tab<LAY>& T, Reader& rd, uint32_t& x, bool active,
                                                    StepSyms& s) {
    constexpr uint32_t D = Hybrid<LAY>::kND, B = Hybrid<LAY>::kNB;
    if (FULL) active = true;
    uint32_t* e = s.e;
    uint32_t acc = 0;                          // largest symbol: the escape symbol is the largest
    // a direct word's state update; returns the symbol
    auto direct = [&](uint32_t w) {
        const uint32_t h = x >> 12;
        if (active) x = (w & 4095u) * h + (h + (w >> 20));
        return (w >> 12) & 255u;
    };
    uint32_t c;
    {
        const uint32_t slot = x & 4095u;
        c = slot >= T.split ? 1u : 0u;
        const uint32_t sy = direct(lds_u32<0>(T.base + 4u * slot));
        renorm_step<FULL>(x, rd, active);
        e[0] = sy;
        if (ESC) acc = sy;
    }
    s.c = c;
    const uint32_t bd = T.base + kHDirect + c * (D * kHDirect);    // f2 given c; f3 (f4) follow
#define EP_FIELD13D(j)                                                                        \
    {                                                                                         \
        const uint32_t sy = direct(lds_u32<((j) - 1) * kHDirect>(bd + 4u * (x & 4095u)));     \
        renorm_step<FULL>(x, rd, active);                                                     \
        e[j] = sy;                                                                            \
        if (ESC) acc = max(acc, sy);                                                          \
    }
    if constexpr (D >= 1) EP_FIELD13D(1)
    if constexpr (D >= 2) EP_FIELD13D(2)
    if constexpr (D >= 3) EP_FIELD13D(3)
#undef EP_FIELD13D
    const uint32_t b1 = T.base + Hybrid<LAY>::kL1 + c * (B * kCtxBytes);            // first two-lookup field's bytes
    const uint32_t b2 = T.base + Hybrid<LAY>::kL2 + c * (B * 1024u + kCosetSkew);   // and its entries
#define EP_FIELD13(j)                                                                         \
    {                                                                                         \
        const uint32_t um = x | 0xFFFFF000u;                                                  \
        const uint32_t sy = lds_u8<((j) - 1 - D) * kCtxBytes>((x & 4095u) | b1);              \
        const uint32_t en = lds_u32<((j) - 1 - D) * 1024>(b2 + 4u * sy);                      \
        if (active) x = (en & kE12QMask) * (x >> 12) + (um + (en >> kE12NegCumShift));        \
        renorm_step<FULL>(x, rd, active);                                                     \
        e[j] = sy;                                                                            \
        if (ESC) acc = max(acc, sy);                                                          \
    }
    if constexpr (D < 1) EP_FIELD13(1)
    if constexpr (D < 2) EP_FIELD13(2)
    if constexpr (D < 3) EP_FIELD13(3)
    EP_FIELD13(4) EP_FIELD13(5) EP_FIELD13(6) EP_FIELD13(7)
#undef EP_FIELD13

    s.from_symbols = true;
    if constexpr (ESC) {
#pragma unroll
        for (int j = 0; j < 8; ++j) s.f[j] = 0;
    }
    if (ESC && __any_sync(kFull, active && acc == uint32_t(kEscape))) {
        // escaped fields: the lane's raw words after its renormalisation words, by field
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const bool mine = active && e[j] == uint32_t(kEscape);
            s.f[j] = mine ? int32_t(int16_t(rd.wn)) : int32_t(e[j]) - kAlphabetR;
            rd.consume_if(mine);
        }
        s.from_symbols = false;
    }
}

template <int LAY, bool ESC, bool FULL, class Reader>
__device__ __forceinline__ void step_symbols(const Tab<LAY>& tab, Reader& rd, uint32_t& x, bool active, StepSyms& s) {
    if constexpr (LAY == 10) step_symbols10<ESC, FULL>(tab.t, rd, x, active, s);
    else if constexpr (LAY == 12) step_symbols12<ESC, FULL>(tab, rd, x, active, s);
    else step_symbols_hybrid<LAY, ESC, FULL>(tab, rd, x, active, s);
}

// Symbol s_j of a decoded step (entry layout of the total).
template <int LAY>
__device__ __forceinline__ uint32_t sym_of(uint32_t e, int j) {
    if constexpr (LAY == 10) return (e >> (kEntrySymShift + (j == 7))) & 255u;
    else return e;
}

template <int OUT, bool VEC, bool ESC, int LAY>
__device__ __forceinline__ void step_emit(const Params& p, const StepSyms& s, const Pos& pos) {
    const uint32_t* e = s.e;
    const uint32_t c = s.c;
    const bool from_symbols = !ESC || s.from_symbols;
    int32_t f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = s.f[j];
    if constexpr (OUT == kOutFields) {
        int16_t* o = reinterpret_cast<int16_t*>(pos.optr);
        o[0] = int16_t(c);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            o[1 + j] = int16_t(from_symbols ? int32_t(sym_of<LAY>(e[j], j)) - kAlphabetR : f[j]);
        return;
    } else {
        // y_j = z_j + c/2, the lattice coordinate (z1..z7 = f1..f7, z8 = 2 f8 + parity of z1..z7),
        // comes from a float T_j built from integer bits: T_j = 1.5 * 2^23 + (an integer below
        // 2^22), so one fused multiply-add y = T k - b is exact (T k is a power-of-two scaling and
        // the difference is a small multiple of 1/2); a * y then rounds once.
        constexpr uint32_t kMagic = 0x4B400000u;     // bits of 1.5 * 2^23
        float val[8];
        const float2 a2 = make_float2(pos.a, pos.a);
        // y = T k - b for the pairs (T_1, T_2), (T_3, T_4), (T_5, T_6), (T_7, T_8), then a * y
        auto scale = [&](const uint32_t (&t)[8], float2 k012, float2 b012, float2 k3, float2 b3) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 y = __ffma2_rn(make_float2(__uint_as_float(t[2 * i]), __uint_as_float(t[2 * i + 1])),
                                            i < 3 ? k012 : k3, i < 3 ? b012 : b3);
                const float2 r = __fmul2_rn(y, a2);
                val[2 * i] = r.x;
                val[2 * i + 1] = r.y;
            }
        };
        if (from_symbols) {
            // Without escapes f_j = s_j - 127.  With 10-bit totals s_j sits in bits 10..17 of a
            // field-1..7 entry and s_8 in bits 11..18 of a field-8 entry, so one mask and OR give
            // (with 12-bit totals e_j is s_j, placed by one shift-and-add)
            //   T_j = 1.5 * 2^23 + 1024 s_j + 512 c:               T_j / 1024 - 12415 = s_j - 127 + c/2,
            //   T_8 = 1.5 * 2^23 + 2048 s_8 + 1024 par + 512 c:    T_8 / 1024 - 12542 = z_8 + c/2,
            // with par = (s_1 + ... + s_7 + 1) mod 2 (7 * 127 is odd), the complement of bit 10
            // of t_1 ^ ... ^ t_7.
            uint32_t t[8];
            const uint32_t km = kMagic | (c << 9);
#pragma unroll
            for (int j = 0; j < 7; ++j)
                t[j] = LAY == 10 ? (e[j] & (0xFFu << kEntrySymShift)) | km : e[j] * 1024u + km;
            const uint32_t px = t[0] ^ t[1] ^ t[2] ^ t[3] ^ t[4] ^ t[5] ^ t[6];
            t[7] = (LAY == 10 ? (e[7] & (0xFFu << (kEntrySymShift + 1))) | km : e[7] * 2048u + km) | (~px & 0x400u);
            const float2 k = make_float2(1.0f / 1024, 1.0f / 1024), b = make_float2(-12415.0f, -12415.0f);
            scale(t, k, b, k, make_float2(-12415.0f, -12542.0f));
        } else {
            // a raw field may be as large as 2^15: T_j = 1.5 * 2^23 + 254 + c + 2 z_j, and
            // T_j / 2 - (1.5 * 2^23 + 254) / 2 = z_j + c/2
            constexpr float kHalfBias = 6291583.0f;      // (1.5 * 2^23 + 254) / 2
            uint32_t t[8];
            const int32_t par = (f[0] + f[1] + f[2] + f[3] + f[4] + f[5] + f[6]) & 1;
            f[7] = 2 * f[7] + par;
#pragma unroll
            for (int j = 0; j < 8; ++j) t[j] = uint32_t(int32_t(kMagic + 254u + c) + 2 * f[j]);
            const float2 k = make_float2(0.5f, 0.5f), b = make_float2(-kHalfBias, -kHalfBias);
            scale(t, k, b, k, b);
        }
        if constexpr (VEC) {
            store_vec<OUT>(pos.optr, val);
        } else {
            constexpr int es = OutElem<OUT>::kBytes;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (8 * int64_t(pos.kcol) + i < p.cols) store_one<OUT>(pos.optr + i * es, val[i]);
        }
    }
}


template <int OUT, bool VEC, bool ESC, int LAY, bool FULL, class Reader>
__device__ __forceinline__ void decode_step(const Params& p, const Tab<LAY>& tab, Reader& rd, uint32_t& x, bool active,
                                            const Pos& pos) {
    if (FULL) active = true;
    StepSyms s;
    step_symbols<LAY, ESC, FULL>(tab, rd, x, active, s);
    if (!active) return;
    step_emit<OUT, VEC, ESC, LAY>(p, s, pos);
}

// Decode `n` full steps, two between runaway checks (the tile buffer's slack covers what two
// steps may read past a checked position), moving the output position by `walk` after each.
// Escape-free blobs are software-pipelined: the symbols of step k + 1 are decoded before step k
// is written (blobs with escapes keep one step at a time, whose raw-field path would otherwise
// hold two steps' fields in registers).
template <int OUT, bool VEC, bool ESC, int LAY, class Reader, class Guard, class Step>
__device__ __forceinline__ uint32_t full_run(const Params& p, const Tab<LAY>& tab, Reader& rd, uint32_t& x, Pos& pos,
                                             uint32_t n, Guard in_range, Step walk) {
    if constexpr (ESC) {
        uint32_t k = 0;
        for (; k + 2 <= n; k += 2) {
            if (!__all_sync(kFull, in_range(rd))) return kStOverrun;  // a corrupt tile ran away
            decode_step<OUT, VEC, ESC, LAY, true>(p, tab, rd, x, true, pos);
            walk(pos);
            decode_step<OUT, VEC, ESC, LAY, true>(p, tab, rd, x, true, pos);
            walk(pos);
        }
        if (k < n) {
            if (!__all_sync(kFull, in_range(rd))) return kStOverrun;
            decode_step<OUT, VEC, ESC, LAY, true>(p, tab, rd, x, true, pos);
            walk(pos);
        }
        return 0;
    } else {
    if (n == 0) return 0;
    StepSyms a, b;
    if (!__all_sync(kFull, in_range(rd))) return kStOverrun;
    step_symbols<LAY, ESC, true>(tab, rd, x, true, a);
    uint32_t k = 1;
    for (; k + 2 <= n; k += 2) {
        if (!__all_sync(kFull, in_range(rd))) return kStOverrun;  // a corrupt tile ran away
        step_symbols<LAY, ESC, true>(tab, rd, x, true, b);
        step_emit<OUT, VEC, ESC, LAY>(p, a, pos);
        walk(pos);
        step_symbols<LAY, ESC, true>(tab, rd, x, true, a);
        step_emit<OUT, VEC, ESC, LAY>(p, b, pos);
        walk(pos);
    }
    if (k < n) {
        if (!__all_sync(kFull, in_range(rd))) return kStOverrun;
        step_symbols<LAY, ESC, true>(tab, rd, x, true, b);
        step_emit<OUT, VEC, ESC, LAY>(p, a, pos);
        walk(pos);
        a = b;
    }
    step_emit<OUT, VEC, ESC, LAY>(p, a, pos);
    walk(pos);
    return 0;
    }
}

template <int OUT, bool VEC, bool ESC, int LAY, int WALK, class Reader, class Guard>
__device__ __forceinline__ uint32_t full_steps(const Params& p, const Tab<LAY>& tab, Reader& rd, uint32_t& x, Pos& pos,
                                               uint32_t nfull, Guard in_range) {
    if constexpr (OUT == kOutFields) {
        return full_run<OUT, VEC, ESC, LAY>(p, tab, rd, x, pos, nfull, in_range, [](Pos& s) { s.optr += 32 * 18; });
    } else if constexpr (WALK == kWalkRows32) {
        constexpr int es = OutElem<OUT>::kBytes;
        const uint32_t per_row = p.vec_per_row / kLanes;
        const int64_t wrap = (p.row_stride - 8 * int64_t(p.vec_per_row)) * es;
        uint32_t left = (p.vec_per_row - pos.kcol + kLanes - 1) / kLanes;  // the same for all 32 lanes
        if (per_row < 8) {
            // short rows: one run over the whole tile (the step pipeline does not restart at every
            // row), the row change a warp-uniform branch in the walk
            float a_next = pos.row + 1 < p.rows ? row_factor<OUT>(p, pos.row + 1) : 0.0f;
            return full_run<OUT, VEC, ESC, LAY>(p, tab, rd, x, pos, nfull, in_range, [&](Pos& s) {
                s.optr += 32 * 8 * es;
                if (--left == 0) {
                    left = per_row;
                    s.optr += wrap;
                    ++s.row;
                    s.a = a_next;
                    a_next = s.row + 1 < p.rows ? row_factor<OUT>(p, s.row + 1) : 0.0f;
                }
            });
        }
        // rows of 8 steps or more: one run per row, nothing but the output pointer moving inside it
        for (uint32_t k = 0; k < nfull;) {
            const uint32_t n = min(left, nfull - k);
            const float a_next = pos.row + 1 < p.rows ? row_factor<OUT>(p, pos.row + 1) : 0.0f;
            const uint32_t st =
                full_run<OUT, VEC, ESC, LAY>(p, tab, rd, x, pos, n, in_range, [](Pos& s) { s.optr += 32 * 8 * es; });
            if (st) return st;
            k += n;
            left -= n;
            if (left == 0) {  // the warp moves to the next row
                left = per_row;
                pos.optr += wrap;
                ++pos.row;
                pos.a = a_next;
            }
        }
        return 0;
    } else {
        return full_run<OUT, VEC, ESC, LAY>(p, tab, rd, x, pos, nfull, in_range,
                                       [&p](Pos& s) { advance<OUT, WALK == kWalkWide>(p, s); });
    }
}

// Decode the steps of one tile with a given word reader; returns the status flags of the tile.
// `pos` is the lane's first vector of the tile (first_pos), found by the caller before the tile's
// words arrived.
template <int OUT, bool VEC, bool ESC, int LAY, class Reader, class Guard>
__device__ __forceinline__ uint32_t decode_tile_steps(const Params& p, const Tab<LAY>& tab, Reader& rd, uint32_t& x,
                                                      uint32_t tile, uint32_t lane, Pos pos, Guard in_range) {
    const int64_t per_tile = int64_t(kLanes) * p.steps;
    const int64_t v0 = int64_t(tile) * per_tile;
    const uint32_t nv = uint32_t(min(per_tile, p.n_vectors - v0));
    const uint32_t nfull = nv / kLanes, rem = nv % kLanes;
    uint32_t st;
    if (VEC && OUT != kOutFields && p.vec_per_row % kLanes == 0)
        st = full_steps<OUT, VEC, ESC, LAY, (VEC && OUT != kOutFields) ? kWalkRows32 : kWalkWide>(p, tab, rd, x, pos, nfull,
                                                                                            in_range);
    else if (p.vec_per_row >= uint32_t(kLanes))
        st = full_steps<OUT, VEC, ESC, LAY, kWalkWide>(p, tab, rd, x, pos, nfull, in_range);
    else
        st = full_steps<OUT, VEC, ESC, LAY, kWalkNarrow>(p, tab, rd, x, pos, nfull, in_range);
    if (st) return st;
    if (rem) {
        if (!__all_sync(kFull, in_range(rd))) return kStOverrun;
        decode_step<OUT, VEC, ESC, LAY, false>(p, tab, rd, x, lane < rem, pos);
    }
    return 0;
}

// The CTA's layout inside its dynamic shared memory: shifted so that the table (and so every
// context's 4 KB sub-table) starts on a 4 KB boundary of the shared window, which makes a
// table address one OR of the slot into the sub-table's base.
template <int WARPS, int LAY>
__device__ __forceinline__ Smem<WARPS, LAY>& smem_layout(uint8_t* raw) {
    const uint32_t pad = (kAlignSlack - (smem_u32(raw) & (kAlignSlack - 1))) & (kAlignSlack - 1);
    return *reinterpret_cast<Smem<WARPS, LAY>*>(raw + pad);
}

// The work of CTA `cta` of the `ncta` CTAs that decode one blob.
// BUILD = false: stage the pre-expanded table from p.tables; true: expand it from `ts` in each CTA.
template <int WARPS, int OUT, bool VEC, bool BUILD, bool ESC, int LAY>
__device__ __forceinline__ void decode_ctas(const Params& p, const TableSrc* ts, const Ctl& ctl, uint8_t* smem_raw,
                                            uint32_t cta, uint32_t ncta) {
    Smem<WARPS, LAY>& sm = smem_layout<WARPS, LAY>(smem_raw);
    constexpr uint32_t kBuf = Geo<WARPS, LAY>::kBuf;
    constexpr uint64_t kMaxTile = 1ull << 22;  // above 160 B + 16 regions of 65535 words
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool fwd = (lane & 1) == 0;  // lanes 2p read forward, lanes 2p+1 backward
    uint8_t* buf = sm.tbuf[warp];
    // Launched as a programmatic dependent of the previous decode on the stream, this kernel may
    // start while that one drains: its prologue (barriers, table and first-tile staging) only
    // reads the blob, and it waits for the previous grid before its first global write.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t buf_a = smem_u32(buf);

    if (threadIdx.x == 0) {
        if (!BUILD) mbar_init(&sm.tbar, 1);
        mbar_init(&sm.pbar, 1);
        for (int w = 0; w < WARPS; ++w) mbar_init(&sm.bar[w], 1);
        fence_proxy_async();
    }
    __syncthreads();  // barriers initialised before anyone uses them
    if (!BUILD && threadIdx.x == 0) {
        mbar_expect_tx(&sm.tbar, TableGeo<LAY>::kBytes);
        for (uint32_t o = 0; o < TableGeo<LAY>::kBytes; o += TableGeo<LAY>::kPiece)
            bulk_g2s(sm.tab + o, p.tables + o, TableGeo<LAY>::kPiece, &sm.tbar);
    }

    const uint32_t tile_stride = ncta * WARPS;
    uint32_t tile = cta + ncta * warp;
    uint32_t staged = 0;  // tiles this warp has staged: its barrier's phase parity

    // Byte extent [a, a + n) of tile t inside the stream section.  The offsets come from device
    // memory that may not be the validated blob (the allocation-free entry point reads the
    // caller's copy), so a tile must hold its header and lie inside the stream; one that does not
    // is reported and skipped, never read.
    auto extent = [&](uint32_t t, uint64_t& a, uint32_t& n) {
        const uint64_t a0 = 16ull * __ldg(p.tile_off + t), a1 = 16ull * __ldg(p.tile_off + t + 1);
        const bool ok = a1 >= a0 + kTileHeadBytes && a1 <= p.stream_bytes && a1 - a0 <= kMaxTile;
        a = a0;
        n = ok ? uint32_t(a1 - a0) : 0u;
        return ok;
    };
    // Stage a tile that fits the buffer (one bulk copy), and ask L2 for the warp's next tile.
    auto stage = [&](uint32_t t, uint64_t a, uint32_t n) {
        __syncwarp();
        if (lane == 0) {
            fence_proxy_async();  // the previous tile's reads of the buffer come first
            mbar_expect_tx(&sm.bar[warp], n);
            bulk_g2s(buf, p.stream + a, n, &sm.bar[warp]);
            const uint32_t nt = t + tile_stride;
            if (nt < p.n_tiles) {
                const uint64_t n0 = 16ull * __ldg(p.tile_off + nt), n1 = 16ull * __ldg(p.tile_off + nt + 1);
                if (n1 > n0 && n1 <= p.stream_bytes)
                    prefetch_l2(p.stream + n0, uint32_t(min(n1 - n0, uint64_t(kBuf))));
            }
        }
    };

    uint64_t t0 = 0;
    uint32_t tbytes = 0;
    bool first_ok = false, first_staged = false;
    if (BUILD) {  // expand the table first: its scratch lies in the tile buffers
        build_tables<WARPS, LAY>(sm.tab, *reinterpret_cast<BuildScratch*>(&sm.tbuf[0][0]), *ts);
        __syncthreads();
    }
    if (tile < p.n_tiles) {  // the first tile's fetch overlaps the table staging
        first_ok = extent(tile, t0, tbytes);
        if (first_ok && tbytes <= kBuf) {
            stage(tile, t0, tbytes);
            first_staged = true;
        }
    }
    if (!BUILD && ctl.probe_tx) {
        // Test only: a wait for bytes that no copy delivers gives up after ctl.wait_spins tries and
        // reports it; the real copies are then waited for (they land) and the CTA leaves.
        if (threadIdx.x == 0) mbar_expect_tx(&sm.pbar, ctl.probe_tx);
        if (!mbar_wait(&sm.pbar, 0, ctl.wait_spins) && lane == 0) atomicOr(p.status, kStTimeout);
        mbar_wait(&sm.tbar, 0);
        goto drain;
    }
    if (!BUILD && !mbar_wait(&sm.tbar, 0, ctl.wait_spins)) {
        if (lane == 0) atomicOr(p.status, kStTimeout);
        goto drain;
    }

    asm volatile("griddepcontrol.wait;" ::: "memory");  // no-op unless launched as a dependent
    if constexpr (OUT == kOutE4M3Row) {  // the per-row scales, spread over the blob's CTAs
        for (int64_t r = int64_t(cta) * blockDim.x + threadIdx.x; r < p.rows; r += int64_t(ncta) * blockDim.x)
            p.sigma[r] = row_sigma(__ldg(p.alpha + r), __ldg(p.rowmax + r));
    }
    {
        Tab<LAY> tab;
        if constexpr (LAY == 10) {
            tab.t = smem_u32(sm.tab);
        } else if constexpr (is_hybrid(LAY)) {
            tab.base = smem_u32(sm.tab);
            tab.split = p.joint_split;
        } else {
            tab.s1 = smem_u32(sm.tab);
            tab.e2 = smem_u32(sm.tab + kSlotBytes);
            tab.s1split = tab.s1 + p.joint_split;
        }
        bool first = true;
        for (; tile < p.n_tiles; tile += tile_stride) {
            bool ok = first_ok;
            if (!first) {
                ok = extent(tile, t0, tbytes);
                if (ok && tbytes <= kBuf) stage(tile, t0, tbytes);
            }
            first = false;
            if (!ok) {
                if (lane == 0) atomicOr(p.status, kStOverrun);
                continue;
            }
            // the lane's output position and row scale: their global loads overlap the staging
            const Pos pos = first_pos<OUT>(p, int64_t(tile) * kLanes * p.steps + lane);
            const bool in_smem = tbytes <= kBuf;
            const uint8_t* tg = p.stream + t0;
            if (in_smem) {
                if (!mbar_wait(&sm.bar[warp], staged & 1u, ctl.wait_spins)) {
                    if (lane == 0) atomicOr(p.status, kStTimeout);
                    return;  // nothing else is in flight into this warp's buffer
                }
                ++staged;
            }
            // tile header: this lane's state; a warp-shuffle prefix sum over the 16 region
            // word counts gives each lane its region
            uint32_t x, cnt;
            if (in_smem) {
                x = lds_u32(buf_a + 4 * lane);
                cnt = lane < uint32_t(kPairs) ? lds_u16(buf_a + 4 * kLanes + 2 * lane) : 0u;
            } else {
                x = __ldg(reinterpret_cast<const uint32_t*>(tg) + lane);
                cnt = lane < uint32_t(kPairs) ? __ldg(reinterpret_cast<const uint16_t*>(tg + 4 * kLanes) + lane) : 0u;
            }
            uint32_t inc = cnt;
#pragma unroll
            for (int o = 1; o < kPairs; o <<= 1) {
                const uint32_t t = __shfl_up_sync(kFull, inc, o);
                if (lane >= uint32_t(o)) inc += t;
            }
            const uint32_t start = __shfl_sync(kFull, inc - cnt, lane >> 1);
            const uint32_t n_region = __shfl_sync(kFull, cnt, lane >> 1);
            const uint32_t total_words = __shfl_sync(kFull, inc, kPairs - 1);
            const int32_t w0 = fwd ? int32_t(start) : int32_t(start + n_region) - 1;  // first word
            const int32_t o0 = int32_t(kTileHeadBytes) + 2 * w0;                     // byte offset
            uint32_t flags, nread;
            if (in_smem) {
                SmemReader rd;
                rd.wd = fwd ? 2 : -2;
                // (clamped: a corrupt count must not move the first load outside the buffer; for a
                // valid tile only a lane with no words is affected, and it reads nothing)
                rd.wp = buf_a + uint32_t(min(max(o0, 0), int32_t(tbytes) - 2));
                rd.wn = lds_u16(rd.wp);
                const uint32_t wp0 = rd.wp, lo = buf_a, hi = buf_a + kBuf;
                flags = decode_tile_steps<OUT, VEC, ESC, LAY>(p, tab, rd, x, tile, lane, pos,
                                                         [=](const SmemReader& r) { return r.wp - lo <= hi - lo; });
                nread = rd.consumed(wp0);
            } else {
                GlobalReader rd;
                rd.tile = tg;
                rd.wd = fwd ? 2 : -2;
                rd.hi = int32_t(tbytes) - 2;
                rd.off = o0;
                rd.wn = __ldg(reinterpret_cast<const uint16_t*>(tg + min(max(o0, 0), rd.hi)));
                flags = decode_tile_steps<OUT, VEC, ESC, LAY>(p, tab, rd, x, tile, lane, pos,
                                                         [](const GlobalReader&) { return true; });
                nread = rd.consumed(o0);
            }
            // integrity: every state back at 2^16; in every region the two lanes read exactly
            // its words; the regions fill the tile up to < 16 bytes of padding
            if (!(flags & kStOverrun)) {
                if (__any_sync(kFull, x != kStateLow)) flags |= kStState;
                const uint32_t pair_read = nread + __shfl_xor_sync(kFull, nread, 1);
                if (__any_sync(kFull, pair_read != n_region)) flags |= kStLeftover;
                const uint32_t used = uint32_t(kTileHeadBytes) + 2u * total_words;
                if (used > tbytes) flags |= kStOverrun;
                else if (tbytes - used >= 16) flags |= kStLeftover;
            }
            if (lane == 0 && flags) atomicOr(p.status, flags);
        }
    }
    return;

drain:
    // no tile is decoded: wait (bounded) for the first tile's copy before leaving
    if (first_staged) mbar_wait(&sm.bar[warp], 0);
}

// One blob over the whole grid.
template <int WARPS, int OUT, bool VEC, bool BUILD, bool ESC, int LAY>
__global__ void __launch_bounds__(WARPS * 32, 1) decode_kernel(const __grid_constant__ Params p,
                                                               const __grid_constant__ TableSrc ts,
                                                               const __grid_constant__ Ctl ctl) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    decode_ctas<WARPS, OUT, VEC, BUILD, ESC, LAY>(p, &ts, ctl, smem_raw, blockIdx.x, gridDim.x);
}

// A set of blobs (all with frequency totals 2^LAY) in one launch: blob m owns CTAs
// [cta0, cta0 + ncta) and stages only its own table.  Every blob picks its store and escape variant.
template <int WARPS, int OUT, int LAY>
__global__ void __launch_bounds__(WARPS * 32, 1) group_kernel(const __grid_constant__ GroupParams g) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint32_t m = 0;
    while (m + 1 < g.n && blockIdx.x >= g.e[m + 1].cta0) ++m;
    const GroupEntry& e = g.e[m];
    if (blockIdx.x >= e.cta0 + e.ncta) return;  // a CTA beyond the last blob's share
    const uint32_t cta = blockIdx.x - e.cta0;
    const Ctl ctl;
    if (e.vec) {
        if (e.esc) decode_ctas<WARPS, OUT, true, false, true, LAY>(e.p, nullptr, ctl, smem_raw, cta, e.ncta);
        else decode_ctas<WARPS, OUT, true, false, false, LAY>(e.p, nullptr, ctl, smem_raw, cta, e.ncta);
    } else {
        if (e.esc) decode_ctas<WARPS, OUT, false, false, true, LAY>(e.p, nullptr, ctl, smem_raw, cta, e.ncta);
        else decode_ctas<WARPS, OUT, false, false, false, LAY>(e.p, nullptr, ctl, smem_raw, cta, e.ncta);
    }
}

// Expands the blob's compact frequency tables into the decode tables (one CTA).
template <int LAY>
struct ExpandSmem {
    alignas(16) uint8_t tab[TableGeo<LAY>::kBytes];
    BuildScratch scratch;
};

template <int WARPS, int LAY>
__global__ void __launch_bounds__(WARPS * 32, 1) expand_tables_kernel(const __grid_constant__ TableSrc p,
                                                                       uint8_t* tables) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    ExpandSmem<LAY>& sm = *reinterpret_cast<ExpandSmem<LAY>*>(smem_raw);
    build_tables<WARPS, LAY>(sm.tab, sm.scratch, p);
    __syncthreads();
    const uint4* s = reinterpret_cast<const uint4*>(sm.tab);
    uint4* d = reinterpret_cast<uint4*>(tables);
    for (uint32_t i = threadIdx.x; i < TableGeo<LAY>::kBytes / 16; i += blockDim.x) d[i] = s[i];
}

// ---- launch functions (host side) ------------------------------------------------------------
// Largest occupancy-limited grid of kernel `fn` on device c (persistent: one wave of CTAs),
// cached per device; 0 when the kernel cannot be configured.
template <class Fn>
int ctas_per_sm(Fn fn, int threads, size_t smem, const LaunchCtx& c, int* cache, std::mutex& mu) {
    std::lock_guard<std::mutex> g(mu);
    if (cache[c.device] == 0) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess) return 0;
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess || n < 1) return 0;
        cache[c.device] = n;
    }
    return cache[c.device];
}

template <int WARPS, int OUT, bool VEC, bool ESC, int LAY>
int launch_one(const Params& p, const Ctl& ctl, cudaStream_t st, const LaunchCtx& c, bool dependent) {
    auto fn = decode_kernel<WARPS, OUT, VEC, false, ESC, LAY>;
    const size_t smem = sizeof(Smem<WARPS, LAY>) + kAlignSlack;
    static std::mutex mu;
    static int per_sm[kMaxDevices] = {};
    const int n = ctas_per_sm(fn, WARPS * 32, smem, c, per_sm, mu);
    if (n == 0) return set_error(EP_ERR_CUDA, "decode kernel: cannot configure its shared memory or occupancy");
    const uint32_t grid = uint32_t(std::min<int64_t>(int64_t(c.sms) * n, p.n_tiles));
    // A dependent launch may begin while the previous kernel on the stream drains (the kernel
    // waits for it before writing); used only when the previous work is another decode.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    const TableSrc none = {};  // the table is pre-expanded
    cudaError_t e = cudaLaunchKernelEx(&cfg, fn, p, none, ctl);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(EP_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
    return EP_OK;
}

template <int WARPS, int OUT, bool ESC, int LAY>
int launch_vec(const Params& p, bool vec, const Ctl& ctl, cudaStream_t st, const LaunchCtx& c, bool dep) {
    return vec ? launch_one<WARPS, OUT, true, ESC, LAY>(p, ctl, st, c, dep)
               : launch_one<WARPS, OUT, false, ESC, LAY>(p, ctl, st, c, dep);
}

template <int OUT, bool ESC, int LAY>
int launch_width(const Params& p, bool vec, int warps, const Ctl& ctl, cudaStream_t st, const LaunchCtx& c, bool dep) {
    if constexpr (LAY != 13 && LAY != 14) {  // layout 13 leaves room for 16 or 20 warps, layout 14 for 16
        if (warps == kWarpsWide) return launch_vec<kWarpsWide, OUT, ESC, LAY>(p, vec, ctl, st, c, dep);
        if (warps == kWarpsMid) return launch_vec<kWarpsMid, OUT, ESC, LAY>(p, vec, ctl, st, c, dep);
    }
    if constexpr (LAY != 14)
        if (warps == kWarps20) return launch_vec<kWarps20, OUT, ESC, LAY>(p, vec, ctl, st, c, dep);
    return launch_vec<kWarpsNarrow, OUT, ESC, LAY>(p, vec, ctl, st, c, dep);
}

template <int OUT, int LAY>
int launch_esc(const Params& p, bool vec, int warps, bool esc, const Ctl& ctl, cudaStream_t st, const LaunchCtx& c,
               bool dep) {
    if constexpr (OUT == kOutFields) {  // test hook: the 16-warp kernel has the registers it needs
        return launch_one<kWarpsNarrow, kOutFields, false, true, LAY>(p, ctl, st, c, false);
    } else {
        return esc ? launch_width<OUT, true, LAY>(p, vec, warps, ctl, st, c, dep)
                   : launch_width<OUT, false, LAY>(p, vec, warps, ctl, st, c, dep);
    }
}

template <int WARPS, int OUT, int LAY>
int group_launch_one(const GroupParams& g, uint32_t grid, cudaStream_t st, const LaunchCtx& c) {
    auto fn = group_kernel<WARPS, OUT, LAY>;
    const size_t smem = sizeof(Smem<WARPS, LAY>) + kAlignSlack;
    static std::mutex mu;
    static int per_sm[kMaxDevices] = {};
    if (ctas_per_sm(fn, WARPS * 32, smem, c, per_sm, mu) == 0)
        return set_error(EP_ERR_CUDA, "group kernel: cannot configure its shared memory or occupancy");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(WARPS * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, fn, g);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(EP_ERR_CUDA, std::string("group launch: ") + cudaGetErrorString(e));
    return EP_OK;
}

// A set of blobs (one total width pb) over `grid` CTAs.
template <int OUT, int LAY>
int group_width(const GroupParams& g, uint32_t grid, int warps, cudaStream_t st, const LaunchCtx& c) {
    if constexpr (LAY != 13 && LAY != 14) {
        if (warps == kWarpsWide) return group_launch_one<kWarpsWide, OUT, LAY>(g, grid, st, c);
        if (warps == kWarpsMid) return group_launch_one<kWarpsMid, OUT, LAY>(g, grid, st, c);
    }
    if constexpr (LAY != 14)
        if (warps == kWarps20) return group_launch_one<kWarps20, OUT, LAY>(g, grid, st, c);
    return group_launch_one<kWarpsNarrow, OUT, LAY>(g, grid, st, c);
}

// The allocation-free decode: tables expanded in every CTA, the status word in caller-provided
// device memory.  Error messages are static strings (no allocation).
template <int WARPS, int OUT, bool VEC, bool ESC, int LAY>
int noalloc_launch_one(const Params& p, const TableSrc& ts, cudaStream_t st, const LaunchCtx& c) {
    auto fn = decode_kernel<WARPS, OUT, VEC, true, ESC, LAY>;
    const size_t smem = sizeof(Smem<WARPS, LAY>) + kAlignSlack;
    static std::mutex mu;
    static int per_sm[kMaxDevices] = {};
    const int n = ctas_per_sm(fn, WARPS * 32, smem, c, per_sm, mu);
    if (n == 0) return set_error_static(EP_ERR_CUDA, "ep_decompress_noalloc: decode kernel does not fit on an SM");
    const uint32_t grid = uint32_t(std::min<int64_t>(int64_t(c.sms) * n, p.n_tiles));
    const Ctl ctl;
    fn<<<grid, WARPS * 32, smem, st>>>(p, ts, ctl);
    if (cudaGetLastError() != cudaSuccess)
        return set_error_static(EP_ERR_CUDA, "ep_decompress_noalloc: kernel launch failed");
    return EP_OK;
}

template <int OUT, int LAY>
int noalloc_esc(const Params& p, const TableSrc& ts, bool vec, bool esc, cudaStream_t st, const LaunchCtx& c) {
    if (esc)
        return vec ? noalloc_launch_one<kWarpsNarrow, OUT, true, true, LAY>(p, ts, st, c)
                   : noalloc_launch_one<kWarpsNarrow, OUT, false, true, LAY>(p, ts, st, c);
    return vec ? noalloc_launch_one<kWarpsNarrow, OUT, true, false, LAY>(p, ts, st, c)
               : noalloc_launch_one<kWarpsNarrow, OUT, false, false, LAY>(p, ts, st, c);
}

// The launch table of one output container and one table layout (each unit compiled from
// decode_unit.cu defines one).  esc: the blob's tables give the escape symbol a frequency (else
// the escape-free kernel runs).
template <int OUT, int LAY>
int unit_single(const Params& p, bool vec, int warps, bool esc, const Ctl& ctl, cudaStream_t st, const LaunchCtx& c,
                bool dep) {
    return launch_esc<OUT, LAY>(p, vec, warps, esc, ctl, st, c, dep);
}
template <int OUT, int LAY>
int unit_group(const GroupParams& g, uint32_t grid, int warps, cudaStream_t st, const LaunchCtx& c) {
    return group_width<OUT, LAY>(g, grid, warps, st, c);
}
template <int OUT, int LAY>
int unit_noalloc(const Params& p, const TableSrc& ts, bool vec, bool esc, cudaStream_t st, const LaunchCtx& c) {
    return noalloc_esc<OUT, LAY>(p, ts, vec, esc, st, c);
}
template <int OUT, int LAY>
constexpr Launchers make_launchers() {
    if constexpr (OUT == kOutFields || OUT == kOutE4M3Row) return Launchers{&unit_single<OUT, LAY>, nullptr, nullptr};
    else if constexpr (LAY == 14) return Launchers{&unit_single<OUT, LAY>, &unit_group<OUT, LAY>, nullptr};
    else return Launchers{&unit_single<OUT, LAY>, &unit_group<OUT, LAY>, &unit_noalloc<OUT, LAY>};
}

}  // namespace
}  // namespace dec
}  // namespace ep
