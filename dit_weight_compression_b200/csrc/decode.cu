// decode.cu -- the GPU entry points of the C ABI: device copies of a blob and its decode tables,
// the decode launches (ep_decompress, ep_decompress_group, ep_decompress_fp8_rowscaled,
// ep_decode_fields), the host-output path, the status word, the launch-shape query and the
// allocation-free decode.  The kernels themselves are in decode_device.cuh; the instantiations of
// each (output container, table layout) pair are compiled from decode_unit.cu.
#include "decode_device.cuh"

#include <numeric>
#include <string>
#include <vector>

// Scratch of ep_decompress_noalloc: a fixed 256-byte array on every device that loads this
// library, held until the process exits.  Host code must not use this name as an address; the
// entry point looks up its device address with cudaGetSymbolAddress.
#define EP_NOALLOC_SCRATCH_WORDS 64
static __device__ __align__(256) uint32_t ep_noalloc_scratch[EP_NOALLOC_SCRATCH_WORDS];

namespace ep {
namespace dec {
namespace {

struct DevInfo {
    bool ready = false;
    int sms = 0;
    cudaStream_t copyback = nullptr;  // host-output path: downloads run here (made on first use,
                                      // kept for the life of the process)
};
std::mutex g_dev_mu;
DevInfo g_dev[kMaxDevices];

static_assert(sizeof(DeviceCopy::tables) / sizeof(DeviceCopy::tables[0]) == kLayouts,
              "one table block per table layout");

// The table layout of a blob's decodes on device `dev` (its SM count known: current_device ran).
int blob_layout(const BlobLayout& L, int dev) {
    return table_layout(L.prob_bits, L.max_tile_bytes, L.n_tiles, g_dev[dev].sms, true);
}

// One blob, with the tables of its own layout (p.tables): 16-warp CTAs when they hold every tile
// at once, else the widest whose buffers hold the largest tile.
int launch(const Params& p, int out_kind, const BlobLayout& L, bool vec, const Ctl& ctl, cudaStream_t st, int device,
           bool dependent) {
    const LaunchCtx c{device, g_dev[device].sms};
    const int lay = blob_layout(L, device);
    const int warps = cta_warps(lay, L.max_tile_bytes, p.n_tiles, uint64_t(c.sms));
    const Launchers* ln = unit_launchers(out_kind, lay);
    if (!ln || !ln->single) return set_error(EP_ERR_DTYPE, "decode: unsupported output container");
    return ln->single(p, vec, warps, L.has_escape != 0, ctl, st, c, dependent);
}

// Share `ctas` CTAs among blobs with tiles[i] tiles: every blob gets one, then each further CTA
// goes to the blob with the most tiles per CTA (lowest index on ties), never more CTAs than tiles.
std::vector<uint32_t> share_ctas(const std::vector<uint32_t>& tiles, uint32_t ctas) {
    std::vector<uint32_t> g(tiles.size(), 1);
    for (uint32_t left = ctas > tiles.size() ? ctas - uint32_t(tiles.size()) : 0; left; --left) {
        int best = -1;
        for (size_t i = 0; i < tiles.size(); ++i) {
            if (g[i] >= tiles[i]) continue;
            if (best < 0 || uint64_t(tiles[i]) * g[best] > uint64_t(tiles[best]) * g[i]) best = int(i);
        }
        if (best < 0) break;
        ++g[best];
    }
    return g;
}

int out_kind_of(int dtype) {
    switch (dtype) {
        case kBF16: return kOutBF16;
        case kFP16: return kOutFP16;
        case kE4M3: return kOutE4M3;
        case kF32: return kOutF32;
        case kI8: return kOutI8;
        default: return -1;
    }
}

#define EP_CUDA(call, what)                                                                      \
    do {                                                                                         \
        cudaError_t e_ = (call);                                                                 \
        if (e_ != cudaSuccess) return set_error(EP_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e_)); \
    } while (0)

int current_device(int& dev) {
    EP_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return set_error(EP_ERR_ARG, "device ordinal out of range");
    std::lock_guard<std::mutex> g(g_dev_mu);
    if (!g_dev[dev].ready) {
        EP_CUDA(cudaDeviceGetAttribute(&g_dev[dev].sms, cudaDevAttrMultiProcessorCount, dev), "SM count");
        g_dev[dev].ready = true;
    }
    return EP_OK;
}

Params make_params(const ep_blob* b, const uint8_t* dblob, const uint8_t* tables, void* out, int64_t row_stride,
                   uint32_t* status) {
    const BlobLayout& L = b->layout;
    Params p;
    p.tables = tables;
    p.tile_off = reinterpret_cast<const uint32_t*>(dblob + L.off_offsets);
    p.stream = dblob + L.off_stream;
    p.alpha = reinterpret_cast<const float*>(dblob + L.off_alpha);
    p.rowmax = reinterpret_cast<const uint16_t*>(dblob + L.off_rowmax);
    p.sigma = nullptr;
    p.out = out;
    p.status = status;
    p.rows = L.rows;
    p.cols = L.cols;
    p.row_stride = row_stride;
    p.n_vectors = L.n_vectors;
    p.stream_bytes = L.total - L.off_stream;
    p.vec_per_row = uint32_t(L.vec_per_row);
    p.steps = L.steps;
    p.n_tiles = L.n_tiles;
    p.joint_split = L.joint_split;
    return p;
}

TableSrc make_tablesrc(const ep_blob* b, const uint8_t* dblob) {
    const BlobLayout& L = b->layout;
    TableSrc t;
    t.blob = dblob;
    for (int c = 0; c < kFieldContexts; ++c) {
        t.q_off[c] = L.q_offset[c];
        t.esc_q[c] = L.esc_q[c];
        t.lo[c] = L.lo[c];
        t.n[c] = L.n[c];
    }
    return t;
}

// The decode tables of layout `lay` in the device copy on `dev`, expanded on first use (one
// allocation, one kernel on `st`, one synchronisation of `st`).  Call with b->mu held, after the
// blob itself is on the device.
int tables_locked(ep_blob* b, int dev, int lay, cudaStream_t st, const uint8_t*& out) {
    DeviceCopy& d = b->dev[dev];
    uint8_t*& slot = d.tables[layout_index(lay)];
    if (!slot) {
        uint8_t* tables = nullptr;
        if (cudaMalloc(&tables, table_bytes(lay)) != cudaSuccess) {
            cudaGetLastError();
            return set_error(EP_ERR_OOM, "decode tables");
        }
        const TableSrc ts = make_tablesrc(b, d.blob);
        auto fn = lay == 10   ? expand_tables_kernel<kWarpsWide, 10>
                  : lay == 11 ? expand_tables_kernel<kWarpsWide, 11>
                  : lay == 12 ? expand_tables_kernel<kWarpsWide, 12>
                  : lay == 13 ? expand_tables_kernel<kWarpsWide, 13>
                  : lay == 14 ? expand_tables_kernel<kWarpsWide, 14> : expand_tables_kernel<kWarpsWide, 15>;
        const size_t smem = lay == 10   ? sizeof(ExpandSmem<10>)
                            : lay == 11 ? sizeof(ExpandSmem<11>)
                            : lay == 12 ? sizeof(ExpandSmem<12>)
                            : lay == 13 ? sizeof(ExpandSmem<13>)
                            : lay == 14 ? sizeof(ExpandSmem<14>) : sizeof(ExpandSmem<15>);
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e == cudaSuccess) {
            fn<<<1, kWarpsWide * 32, smem, st>>>(ts, tables);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) {
            cudaFree(tables);
            return set_error(EP_ERR_CUDA, std::string("table expansion: ") + cudaGetErrorString(e));
        }
        slot = tables;
    }
    out = slot;
    return EP_OK;
}

// Device copy of the blob, its status word and the tables of the layout its own decodes use on
// `dev` (allocated and filled on first use).
int ensure_device(ep_blob* b, int dev, cudaStream_t st) {
    std::lock_guard<std::mutex> g(b->mu);
    DeviceCopy& d = b->dev[dev];
    if (!d.blob) {
        uint8_t* blob = nullptr;
        uint32_t* status = nullptr;
        if (cudaMalloc(&blob, b->bytes.size()) != cudaSuccess || cudaMalloc(&status, 16) != cudaSuccess) {
            cudaFree(blob);
            cudaFree(status);
            cudaGetLastError();
            return set_error(EP_ERR_OOM, "device copy of the blob");
        }
        cudaError_t e = cudaMemcpyAsync(blob, b->bytes.data(), b->bytes.size(), cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, 16, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) {
            cudaFree(blob);
            cudaFree(status);
            return set_error(EP_ERR_CUDA, std::string("blob upload: ") + cudaGetErrorString(e));
        }
        d.blob = blob;
        d.status = status;
    }
    const uint8_t* t = nullptr;
    return tables_locked(b, dev, blob_layout(b->layout, dev), st, t);
}

// The device copy on `dev` and its tables of layout `lay`.
int ensure_tables(ep_blob* b, int dev, int lay, cudaStream_t st, const uint8_t*& out) {
    int rc = ensure_device(b, dev, st);
    if (rc != EP_OK) return rc;
    std::lock_guard<std::mutex> g(b->mu);
    return tables_locked(b, dev, lay, st, out);
}

// Blob-owned staging buffers of the host-output path on `dev`: the per-call upload target, the
// decoded output (at least out_bytes) and, for the row-scaled FP8 container, the row scales.
int ensure_staging(ep_blob* b, int dev, size_t out_bytes, bool sigma) {
    std::lock_guard<std::mutex> g(b->mu);
    DeviceCopy& d = b->dev[dev];
    if (!d.stage_blob && cudaMalloc(&d.stage_blob, b->bytes.size()) != cudaSuccess)
        return set_error(EP_ERR_OOM, "host-output decode: staging copy of the blob");
    if (d.stage_out_bytes < out_bytes) {
        cudaFree(d.stage_out);
        d.stage_out = nullptr;
        d.stage_out_bytes = 0;
        if (cudaMalloc(&d.stage_out, out_bytes) != cudaSuccess)
            return set_error(EP_ERR_OOM, "host-output decode: staging output");
        d.stage_out_bytes = out_bytes;
    }
    if (sigma && !d.stage_sigma && cudaMalloc(&d.stage_sigma, 4 * size_t(b->layout.rows)) != cudaSuccess)
        return set_error(EP_ERR_OOM, "host-output decode: staging row scales");
    for (cudaEvent_t& e : d.chunk_done)
        if (!e && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
            e = nullptr;
            cudaGetLastError();
            return set_error(EP_ERR_CUDA, "host-output decode: chunk events");
        }
    if (!b->host_pinned) {
        // best effort: page-locked host bytes make the per-call upload a direct DMA
        if (cudaHostRegister(b->bytes.data(), b->bytes.size(), cudaHostRegisterDefault) == cudaSuccess)
            b->host_pinned = true;
        else
            cudaGetLastError();
    }
    return EP_OK;
}

bool vec_ok(const BlobLayout& L, const void* out, int64_t row_stride, int dtype) {
    const uintptr_t align = (dtype == kE4M3 || dtype == kI8) ? 8 : 16;
    return L.cols % 8 == 0 && row_stride % 8 == 0 && (reinterpret_cast<uintptr_t>(out) % align) == 0;
}

// ---- host-output path ------------------------------------------------------------------------
constexpr size_t kHostChunkBytes = size_t(4) << 20;  // output bytes per chunk, at least

// The device's copy-back stream.
int copyback_stream(int dev, cudaStream_t& out) {
    std::lock_guard<std::mutex> g(g_dev_mu);
    if (!g_dev[dev].copyback)
        EP_CUDA(cudaStreamCreateWithFlags(&g_dev[dev].copyback, cudaStreamNonBlocking), "copy-back stream");
    out = g_dev[dev].copyback;
    return EP_OK;
}

// Tile boundaries of the host-output pipeline: chunk i holds tiles [t[i], t[i+1]).  Every chunk
// starts on a row (its first vector is a multiple of the row's vector count), carries at least
// kHostChunkBytes of output where the blob has that much, and there are at most kMaxHostChunks.
// A small blob, or one whose tiles end on a row boundary only rarely, is one chunk.
std::vector<uint32_t> host_chunks(const BlobLayout& L, size_t out_bytes) {
    std::vector<uint32_t> t{0};
    const uint64_t per = uint64_t(kLanes) * L.steps;                       // vectors per tile
    const uint64_t vpr = uint64_t(L.vec_per_row);
    const uint64_t unit = vpr / std::gcd(per, vpr);                        // tiles per row-aligned unit
    const uint64_t n = std::min<uint64_t>(kMaxHostChunks, out_bytes / kHostChunkBytes);
    if (n >= 2 && unit < L.n_tiles) {
        const uint64_t units = (uint64_t(L.n_tiles) + unit - 1) / unit;
        for (uint64_t i = 1; i < n; ++i) {
            const uint64_t b = (units * i / n) * unit;
            if (b > t.back() && b < L.n_tiles) t.push_back(uint32_t(b));
        }
    }
    t.push_back(L.n_tiles);
    return t;
}

// Decode into host memory (out->device == -1) and, for the row-scaled FP8 container, host row
// scales.  The bytes before the stream section go up first; then chunk by chunk (whole rows
// each), the chunk's stream bytes are uploaded and its tiles decoded on `st`, and the copy-back
// stream waits for that decode and downloads the chunk's rows.  So the download of one chunk
// overlaps the upload and decode of the next, and a call costs about its longer copy direction
// instead of the sum of both.  A chunk is decoded as the blob restricted to its rows: the tile
// offsets, scales, row maxima and output start at the chunk's first tile and row, which every
// tile's decode already treats as its own origin.  Returns when every row is back.
int decode_to_host(ep_blob* b, const ep_tensor* out, int kind, float* host_sigma, cudaStream_t st, int dev,
                   const char* what) {
    const BlobLayout& L = b->layout;
    const size_t es = size_t(dtype_bytes(out->dtype));
    const size_t row_bytes = size_t(L.cols) * es;
    const uint8_t* tables = nullptr;
    int rc = ensure_tables(b, dev, blob_layout(L, dev), st, tables);
    if (rc == EP_OK) rc = ensure_staging(b, dev, row_bytes * size_t(L.rows), host_sigma != nullptr);
    cudaStream_t cb = nullptr;
    if (rc == EP_OK) rc = copyback_stream(dev, cb);
    if (rc != EP_OK) return rc;
    const DeviceCopy& d = b->dev[dev];
    const uint8_t* host = b->bytes.data();
    const uint64_t stream_total = L.total - L.off_stream;
    const uint64_t per = uint64_t(kLanes) * L.steps;
    const std::vector<uint32_t> t = host_chunks(L, row_bytes * size_t(L.rows));
    const std::string w(what);
    // Everything is issued first; whatever happens, both streams are drained before returning, so
    // no download of an earlier chunk is still writing into the caller's buffer after an error.
    auto issue = [&]() -> int {
        EP_CUDA(cudaMemcpyAsync(d.stage_blob, host, L.off_stream, cudaMemcpyHostToDevice, st), w + ": upload");
        uint64_t up = 0;  // stream bytes uploaded so far
        for (size_t i = 0; i + 1 < t.size(); ++i) {
            const uint32_t t0 = t[i], t1 = t[i + 1];
            const bool last = i + 2 == t.size();
            // tile offsets are checked to rise to the stream's end, so chunk i's tiles lie in [0, end)
            const uint64_t end =
                last ? stream_total : std::min<uint64_t>(stream_total, 16ull * rd32(host + L.off_offsets + 4ull * t1));
            if (end > up) {
                EP_CUDA(cudaMemcpyAsync(d.stage_blob + L.off_stream + up, host + L.off_stream + up, end - up,
                                        cudaMemcpyHostToDevice, st),
                        w + ": upload");
                up = end;
            }
            const int64_t v0 = int64_t(t0) * int64_t(per);
            const int64_t v1 = last ? L.n_vectors : int64_t(t1) * int64_t(per);
            const int64_t r0 = v0 / L.vec_per_row, r1 = last ? L.rows : v1 / L.vec_per_row;
            uint8_t* dout = d.stage_out + size_t(r0) * row_bytes;
            Params p = make_params(b, d.stage_blob, tables, dout, L.cols, d.status);
            p.tile_off += t0;
            p.alpha += r0;
            p.rowmax += r0;
            p.rows = r1 - r0;
            p.n_vectors = v1 - v0;
            p.n_tiles = t1 - t0;
            if (host_sigma) p.sigma = d.stage_sigma + r0;
            const int lrc = launch(p, kind, L, vec_ok(L, dout, L.cols, out->dtype), Ctl(), st, dev, false);
            if (lrc != EP_OK) return lrc;
            EP_CUDA(cudaEventRecord(d.chunk_done[i], st), w + ": chunk event");
            EP_CUDA(cudaStreamWaitEvent(cb, d.chunk_done[i], 0), w + ": chunk wait");
            uint8_t* hout = static_cast<uint8_t*>(out->data) + size_t(r0) * size_t(out->row_stride) * es;
            if (out->row_stride == L.cols)  // contiguous rows: one linear copy
                EP_CUDA(cudaMemcpyAsync(hout, dout, size_t(r1 - r0) * row_bytes, cudaMemcpyDeviceToHost, cb),
                        w + ": download");
            else
                EP_CUDA(cudaMemcpy2DAsync(hout, size_t(out->row_stride) * es, dout, row_bytes, row_bytes,
                                          size_t(r1 - r0), cudaMemcpyDeviceToHost, cb),
                        w + ": download");
        }
        if (host_sigma)
            EP_CUDA(cudaMemcpyAsync(host_sigma, d.stage_sigma, 4 * size_t(L.rows), cudaMemcpyDeviceToHost, cb),
                    w + ": download");
        return EP_OK;
    };
    rc = issue();
    const cudaError_t e1 = cudaStreamSynchronize(cb), e2 = cudaStreamSynchronize(st);
    if (rc != EP_OK) return rc;
    if (e1 != cudaSuccess || e2 != cudaSuccess)
        return set_error(EP_ERR_CUDA, w + ": synchronise: " + cudaGetErrorString(e1 != cudaSuccess ? e1 : e2));
    return EP_OK;
}

// ---- allocation-free decode (ep_decompress_noalloc) -------------------------------------------
// The decode kernel's only scratch is its 4-byte status word.  For callers that may not allocate,
// that word lives in the file-scope array above instead of blob-owned device memory.
constexpr int kNoallocScratchWords = EP_NOALLOC_SCRATCH_WORDS;  // 256 bytes; a launch uses word 0

struct NoallocDevice {
    bool ready = false;
    uint32_t* scratch = nullptr;  // device address of ep_noalloc_scratch on this device
    int sms = 0;
};
NoallocDevice g_noalloc[kMaxDevices];
std::mutex g_noalloc_mu;

}  // namespace
}  // namespace dec
}  // namespace ep

using namespace ep;
using namespace ep::dec;

extern "C" int ep_blob_prepare(ep_blob* b, int device, void* stream) {
    clear_error();
    if (!b) return set_error(EP_ERR_ARG, "ep_blob_prepare: NULL blob");
    int prev = 0;
    EP_CUDA(cudaGetDevice(&prev), "cudaGetDevice");
    EP_CUDA(cudaSetDevice(device), "cudaSetDevice");
    int dev = 0;
    int rc = current_device(dev);
    if (rc == EP_OK) rc = ensure_device(b, dev, static_cast<cudaStream_t>(stream));
    cudaSetDevice(prev);
    return rc;
}

extern "C" int ep_decompress(const ep_blob* cb, const ep_tensor* out, void* stream) {
    clear_error();
    if (!cb || !out || !out->data) return set_error(EP_ERR_ARG, "ep_decompress: NULL argument");
    ep_blob* b = const_cast<ep_blob*>(cb);
    const BlobLayout& L = b->layout;
    const int kind = out_kind_of(out->dtype);
    if (kind < 0) return set_error(EP_ERR_DTYPE, "ep_decompress: unsupported output dtype");
    if (out->rows != L.rows || out->cols != L.cols)
        return set_error(EP_ERR_SHAPE, "ep_decompress: output shape differs from the blob's");
    if (out->row_stride < out->cols) return set_error(EP_ERR_ARG, "ep_decompress: row_stride < cols");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    int rc = current_device(dev);
    if (rc != EP_OK) return rc;

    if (out->device >= 0) {
        if (out->device != dev)
            return set_error(EP_ERR_ARG, "ep_decompress: output is not on the current device");
        const uint8_t* tables = nullptr;
        rc = ensure_tables(b, dev, blob_layout(L, dev), st, tables);
        if (rc != EP_OK) return rc;
        const DeviceCopy& d = b->dev[dev];
        const bool vec = vec_ok(L, out->data, out->row_stride, out->dtype);
        Params p = make_params(b, d.blob, tables, out->data, out->row_stride, d.status);
        return launch(p, kind, L, vec, Ctl(), st, dev, true);
    }

    return decode_to_host(b, out, kind, nullptr, st, dev, "ep_decompress");
}

extern "C" int ep_decompress_group(const ep_blob* const* blobs, const ep_tensor* outs, int n, void* stream) {
    clear_error();
    if (n == 0) return EP_OK;
    if (n < 0 || !blobs || !outs) return set_error(EP_ERR_ARG, "ep_decompress_group: NULL argument or n < 0");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    int rc = current_device(dev);
    if (rc != EP_OK) return rc;
    const int dtype = outs[0].dtype;
    const int kind = out_kind_of(dtype);
    if (kind < 0) return set_error(EP_ERR_DTYPE, "ep_decompress_group: unsupported output dtype");
    for (int i = 0; i < n; ++i) {  // validate everything before launching anything
        const ep_tensor& o = outs[i];
        if (!blobs[i] || !o.data) return set_error(EP_ERR_ARG, "ep_decompress_group: NULL blob or output");
        if (o.dtype != dtype) return set_error(EP_ERR_DTYPE, "ep_decompress_group: outputs differ in dtype");
        if (o.device != dev)
            return set_error(EP_ERR_ARG, "ep_decompress_group: outputs must be on the current device");
        const BlobLayout& L = blobs[i]->layout;
        if (o.rows != L.rows || o.cols != L.cols)
            return set_error(EP_ERR_SHAPE, "ep_decompress_group: an output's shape differs from its blob's");
        if (o.row_stride < o.cols) return set_error(EP_ERR_ARG, "ep_decompress_group: row_stride < cols");
    }
    const int sms = g_dev[dev].sms;
    const int chunk = std::max(1, std::min(kMaxGroup, sms));
    // Blobs of one frequency-total width go in chunks of up to `chunk` blobs, one launch each.  A
    // chunk's layout and CTA width follow from its own tile count and largest tile, so every blob
    // of the chunk needs that layout's tables: all are made ready before anything is launched.
    struct Launch {
        std::vector<int> idx;
        int lay = 0, warps = 0;
        uint32_t ctas = 0;
        std::vector<uint32_t> share;
        std::vector<const uint8_t*> tables;
    };
    std::vector<Launch> plan;
    for (int pb : {12, 10}) {
        std::vector<int> idx;
        for (int i = 0; i < n; ++i)
            if (blobs[i]->layout.prob_bits == pb) idx.push_back(i);
        for (size_t c0 = 0; c0 < idx.size(); c0 += size_t(chunk)) {
            Launch l;
            l.idx.assign(idx.begin() + std::ptrdiff_t(c0), idx.begin() + std::ptrdiff_t(std::min(idx.size(), c0 + size_t(chunk))));
            std::vector<uint32_t> tiles;
            uint64_t total = 0, max_tile = 0;
            for (int i : l.idx) {
                const BlobLayout& L = blobs[i]->layout;
                tiles.push_back(L.n_tiles);
                total += L.n_tiles;
                max_tile = std::max<uint64_t>(max_tile, L.max_tile_bytes);
            }
            l.share = share_ctas(tiles, uint32_t(sms));
            for (uint32_t g : l.share) l.ctas += g;
            l.lay = table_layout(pb, max_tile, total, sms, true);
            l.warps = cta_warps(l.lay, max_tile, total, l.ctas);
            for (int i : l.idx) {
                const uint8_t* t = nullptr;
                rc = ensure_tables(const_cast<ep_blob*>(blobs[i]), dev, l.lay, st, t);
                if (rc != EP_OK) return rc;
                l.tables.push_back(t);
            }
            plan.push_back(std::move(l));
        }
    }
    for (const Launch& l : plan) {
        GroupParams gp = {};
        gp.n = uint32_t(l.idx.size());
        uint32_t cta = 0;
        for (size_t k = 0; k < l.idx.size(); ++k) {
            const ep_blob* b = blobs[l.idx[k]];
            const ep_tensor& o = outs[l.idx[k]];
            const DeviceCopy& d = b->dev[dev];
            GroupEntry& e = gp.e[k];
            e.p = make_params(b, d.blob, l.tables[k], o.data, o.row_stride, d.status);
            e.cta0 = cta;
            e.ncta = l.share[k];
            e.vec = vec_ok(b->layout, o.data, o.row_stride, dtype) ? 1u : 0u;
            e.esc = b->layout.has_escape ? 1u : 0u;
            cta += e.ncta;
        }
        const Launchers* ln = unit_launchers(kind, l.lay);
        if (!ln || !ln->group) return set_error(EP_ERR_DTYPE, "ep_decompress_group: unsupported output container");
        rc = ln->group(gp, cta, l.warps, st, LaunchCtx{dev, sms});
        if (rc != EP_OK) return rc;
    }
    return EP_OK;
}

extern "C" int ep_decompress_fp8_rowscaled(const ep_blob* cb, const ep_tensor* out, float* row_scale, void* stream) {
    clear_error();
    if (!cb || !out || !out->data || !row_scale)
        return set_error(EP_ERR_ARG, "ep_decompress_fp8_rowscaled: NULL argument");
    ep_blob* b = const_cast<ep_blob*>(cb);
    const BlobLayout& L = b->layout;
    if (out->dtype != kE4M3) return set_error(EP_ERR_DTYPE, "ep_decompress_fp8_rowscaled: output must be FP8 E4M3");
    if (out->rows != L.rows || out->cols != L.cols)
        return set_error(EP_ERR_SHAPE, "ep_decompress_fp8_rowscaled: output shape differs from the blob's");
    if (out->row_stride < out->cols) return set_error(EP_ERR_ARG, "ep_decompress_fp8_rowscaled: row_stride < cols");
    if (reinterpret_cast<uintptr_t>(row_scale) % 4 != 0)
        return set_error(EP_ERR_ARG, "ep_decompress_fp8_rowscaled: row_scale must be 4-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    int rc = current_device(dev);
    if (rc != EP_OK) return rc;
    if (out->device >= 0) {
        if (out->device != dev)
            return set_error(EP_ERR_ARG, "ep_decompress_fp8_rowscaled: output is not on the current device");
        const uint8_t* tables = nullptr;
        rc = ensure_tables(b, dev, blob_layout(L, dev), st, tables);
        if (rc != EP_OK) return rc;
        const DeviceCopy& d = b->dev[dev];
        const bool vec = vec_ok(L, out->data, out->row_stride, kE4M3);
        Params p = make_params(b, d.blob, tables, out->data, out->row_stride, d.status);
        p.sigma = row_scale;
        return launch(p, kOutE4M3Row, L, vec, Ctl(), st, dev, true);
    }
    return decode_to_host(b, out, kOutE4M3Row, row_scale, st, dev, "ep_decompress_fp8_rowscaled");
}

extern "C" int ep_decode_fields(const ep_blob* cb, int16_t* fields, void* stream) {
    clear_error();
    if (!cb || !fields) return set_error(EP_ERR_ARG, "ep_decode_fields: NULL argument");
    ep_blob* b = const_cast<ep_blob*>(cb);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    int rc = current_device(dev);
    const uint8_t* tables = nullptr;
    if (rc == EP_OK) rc = ensure_tables(b, dev, blob_layout(b->layout, dev), st, tables);
    if (rc != EP_OK) return rc;
    const DeviceCopy& d = b->dev[dev];
    Params p = make_params(b, d.blob, tables, fields, b->layout.cols, d.status);
    return launch(p, kOutFields, b->layout, false, Ctl(), st, dev, false);
}

extern "C" int ep_decode_wait_probe(const ep_blob* cb, uint32_t wait_spins, void* stream) {
    clear_error();
    if (!cb || wait_spins == 0) return set_error(EP_ERR_ARG, "ep_decode_wait_probe: NULL blob or zero limit");
    ep_blob* b = const_cast<ep_blob*>(cb);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int dev = 0;
    int rc = current_device(dev);
    const uint8_t* tables = nullptr;
    if (rc == EP_OK) rc = ensure_tables(b, dev, blob_layout(b->layout, dev), st, tables);
    if (rc != EP_OK) return rc;
    const DeviceCopy& d = b->dev[dev];
    // no tile is decoded and nothing is written: every CTA waits for bytes no copy delivers
    Params p = make_params(b, d.blob, tables, nullptr, b->layout.cols, d.status);
    Ctl ctl;
    ctl.wait_spins = wait_spins;
    ctl.probe_tx = 16;
    return launch(p, kOutFields, b->layout, false, ctl, st, dev, false);
}

extern "C" int ep_decode_shape(const ep_blob* b, int* layout, int* warps) {
    clear_error();
    if (!b || !layout || !warps) return set_error(EP_ERR_ARG, "ep_decode_shape: NULL argument");
    int dev = 0;
    const int rc = current_device(dev);
    if (rc != EP_OK) return rc;
    const BlobLayout& L = b->layout;
    const int lay = blob_layout(L, dev);  // as launch() decides for a whole-blob decode
    *layout = lay;
    *warps = cta_warps(lay, L.max_tile_bytes, L.n_tiles, uint64_t(g_dev[dev].sms));
    return EP_OK;
}

extern "C" int ep_decode_status(const ep_blob* cb, void* stream) {
    clear_error();
    if (!cb) return set_error(EP_ERR_ARG, "ep_decode_status: NULL blob");
    ep_blob* b = const_cast<ep_blob*>(cb);
    int dev = 0;
    int rc = current_device(dev);
    if (rc != EP_OK) return rc;
    DeviceCopy& d = b->dev[dev];
    if (!d.status) return EP_OK;  // never decoded on this device
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t s = 0;
    EP_CUDA(cudaStreamSynchronize(st), "ep_decode_status: synchronise");
    EP_CUDA(cudaMemcpy(&s, d.status, 4, cudaMemcpyDeviceToHost), "ep_decode_status: read");
    EP_CUDA(cudaMemset(d.status, 0, 4), "ep_decode_status: clear");
    if (s == 0) return EP_OK;
    std::string why = "GPU decode found a corrupt blob:";
    if (s & kStOverrun) why += " tile read past its end;";
    if (s & kStState) why += " final rANS state not 2^16;";
    if (s & kStLeftover) why += " unread tile words;";
    if (s & kStTimeout) why += " bulk-copy wait limit reached;";
    return set_error(EP_ERR_CORRUPT, why);
}

extern "C" void ep_blob_free(ep_blob* b) {
    if (!b) return;
    int prev = 0;
    cudaGetDevice(&prev);
    for (int dv = 0; dv < kMaxDevices; ++dv) {
        DeviceCopy& d = b->dev[dv];
        if (!d.blob && !d.stage_blob && !d.stage_out) continue;
        cudaSetDevice(dv);
        cudaFree(d.blob);
        for (uint8_t* t : d.tables) cudaFree(t);
        cudaFree(d.status);
        cudaFree(d.stage_blob);
        cudaFree(d.stage_out);
        cudaFree(d.stage_sigma);
        for (cudaEvent_t e : d.chunk_done)
            if (e) cudaEventDestroy(e);
    }
    if (b->host_pinned) cudaHostUnregister(b->bytes.data());
    cudaSetDevice(prev);
    delete b;
}

extern "C" int ep_decompress_noalloc(const ep_blob* cb, const void* device_blob, size_t device_blob_bytes,
                                     const ep_tensor* out, void* stream, int wait) {
    clear_error();
    if (!cb || !device_blob || !out || !out->data)
        return set_error_static(EP_ERR_ARG, "ep_decompress_noalloc: NULL argument");
    const BlobLayout& L = cb->layout;
    // every offset the kernel follows lies inside the blob's size, so a buffer of at least that
    // many bytes keeps all its reads inside the caller's allocation
    if (device_blob_bytes < L.total)
        return set_error_static(EP_ERR_ARG, "ep_decompress_noalloc: device_blob is smaller than the blob");
    const int kind = out_kind_of(out->dtype);
    if (kind < 0) return set_error_static(EP_ERR_DTYPE, "ep_decompress_noalloc: unsupported output dtype");
    if (out->rows != L.rows || out->cols != L.cols)
        return set_error_static(EP_ERR_SHAPE, "ep_decompress_noalloc: output shape differs from the blob's");
    if (out->row_stride < out->cols)
        return set_error_static(EP_ERR_ARG, "ep_decompress_noalloc: row_stride < cols");
    if (reinterpret_cast<uintptr_t>(device_blob) % 16 != 0)
        return set_error_static(EP_ERR_ARG, "ep_decompress_noalloc: device_blob must be 16-byte aligned");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return set_error_static(EP_ERR_CUDA, "ep_decompress_noalloc: no usable current device");
    if (out->device != dev)
        return set_error_static(EP_ERR_ARG, "ep_decompress_noalloc: output must be device memory on the current device");
    // One status word per launch; the array holds kNoallocScratchWords.
    constexpr int kWordsNeeded = 1;
    static_assert(kWordsNeeded <= kNoallocScratchWords, "scratch array too small");
    {
        // first call on this device: find the array's device address (with this device current)
        std::lock_guard<std::mutex> g(g_noalloc_mu);
        NoallocDevice& nd = g_noalloc[dev];
        if (!nd.ready) {
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, ep_noalloc_scratch) != cudaSuccess || !ptr)
                return set_error_static(EP_ERR_CUDA, "ep_decompress_noalloc: cudaGetSymbolAddress failed");
            if (cudaDeviceGetAttribute(&nd.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return set_error_static(EP_ERR_CUDA, "ep_decompress_noalloc: cannot read the SM count");
            nd.scratch = static_cast<uint32_t*>(ptr);
            nd.ready = true;
        }
    }
    uint32_t* status = g_noalloc[dev].scratch;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the status word must start at zero for this call
    if (cudaMemsetAsync(status, 0, sizeof(uint32_t) * kWordsNeeded, st) != cudaSuccess)
        return set_error_static(EP_ERR_CUDA, "ep_decompress_noalloc: clearing the status word failed");
    const bool vec = vec_ok(L, out->data, out->row_stride, out->dtype);
    Params p = make_params(cb, static_cast<const uint8_t*>(device_blob), nullptr, out->data, out->row_stride,
                           status);
    const TableSrc ts = make_tablesrc(cb, static_cast<const uint8_t*>(device_blob));
    // 16-warp CTAs only, and layouts 10, 12 and 13
    const Launchers* ln = unit_launchers(kind, table_layout(L.prob_bits, L.max_tile_bytes, L.n_tiles, 1, false));
    if (!ln || !ln->noalloc) return set_error_static(EP_ERR_DTYPE, "ep_decompress_noalloc: unsupported output dtype");
    int rc = ln->noalloc(p, ts, vec, L.has_escape != 0, st, LaunchCtx{dev, g_noalloc[dev].sms});
    if (rc != EP_OK || !wait) return rc;
    uint32_t s = 0;
    if (cudaMemcpyAsync(&s, status, sizeof s, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return set_error_static(EP_ERR_CUDA, "ep_decompress_noalloc: reading the status word failed");
    if (s != 0) return set_error_static(EP_ERR_CORRUPT, "ep_decompress_noalloc: GPU decode found a corrupt blob");
    return EP_OK;
}
