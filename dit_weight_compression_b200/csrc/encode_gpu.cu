// encode_gpu.cu -- the encoder on the GPU, for tensors already in device memory.
//
// Same steps and the same bytes as the host encoder ("EntroPack lattice compression",
// documentation page: sections "Lattice quantization and integer fields" and "Rate selection and
// refinement" for the quantiser and the scale search, "Encoding and reconstruction" for the
// tiles), with the parallel work on the device:
//   * row RMS and row least-squares scales: 32 rows per warp; each 32x32 block of elements is
//     staged in shared memory so that loads are coalesced, then every lane adds its row's terms
//     in column order -- the host's summation order, so the doubles come out bit-identical;
//   * lattice quantisation (sampled rows during the scale search, then all rows): one thread per
//     8-vector, E8 nearest point in fp64 with explicitly rounded operations (no contraction), a
//     shared-memory symbol histogram per block;
//   * rANS tiles: one warp per tile and one lane per interleaved state, twice -- a pass that
//     counts each lane's words (giving every tile's size), then, after the host lays the tiles
//     out, a pass that writes each word at its place in the lane's region.
// The host runs what is small or sequential: the 48-step bisection over the scale (each step one
// sampled quantisation on the device), the frequency tables and the blob header (tables.h).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstring>
#include <string>
#include <vector>

#include "format.h"
#include "tables.h"

namespace ep {
namespace {

constexpr uint32_t kFullMask = 0xFFFFFFFFu;
constexpr double kClampT = 32764.0;  // |x_hat / s| clamp: every field fits an int16

// ---- device arithmetic, rounded exactly as the host's fp64 code ---------------------------------
__device__ __forceinline__ double e4m3_value(uint32_t b) {  // OCP E4M3: bias 7, S.1111.111 is NaN
    const int e = (b >> 3) & 0xF;
    const uint32_t m = b & 7;
    double mag = (e == 15 && m == 7) ? __longlong_as_double(0x7FF8000000000000ll)
               : e == 0 ? ldexp(double(m), -9)
               : ldexp(double(m | 8), e - 10);
    return (b & 0x80) ? -mag : mag;
}

// Element idx of a row-major container array, as its exact value.
__device__ __forceinline__ double load_elem(const uint8_t* base, int dtype, int64_t idx) {
    switch (dtype) {
        case kBF16: return double(__uint_as_float(uint32_t(reinterpret_cast<const uint16_t*>(base)[idx]) << 16));
        case kFP16: return double(__half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(base)[idx])));
        case kE4M3: return e4m3_value(base[idx]);
        case kI8: return double(int8_t(base[idx]));
        default: return double(reinterpret_cast<const float*>(base)[idx]);
    }
}

// Conway-Sloane nearest point of D8 (rounding halves away from zero; on an odd sum the coordinate
// rounding disturbed most, first on ties, moves one step toward its value, up when exact).
__device__ __forceinline__ void nearest_d8(const double u[8], double g[8]) {
    long long sum = 0;
    int worst_i = 0;
    double worst = -1.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        g[i] = round(u[i]);
        sum += (long long)g[i];
        const double miss = fabs(__dsub_rn(u[i], g[i]));
        if (miss > worst) { worst = miss; worst_i = i; }
    }
    if (sum % 2 != 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i == worst_i) g[i] = __dadd_rn(g[i], (u[i] < g[i]) ? -1.0 : 1.0);
    }
}

// Nearest point of E8 = D8 u (D8 + 1/2); equal distances keep the integer coset.  Returns the coset.
__device__ __forceinline__ int nearest_e8(const double t[8], double y[8]) {
    double a[8], b[8], u[8];
    nearest_d8(t, a);
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = __dsub_rn(t[i], 0.5);
    nearest_d8(u, b);
    double da = 0.0, db = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        b[i] = __dadd_rn(b[i], 0.5);
        const double ea = __dsub_rn(t[i], a[i]), eb = __dsub_rn(t[i], b[i]);
        da = __dadd_rn(da, __dmul_rn(ea, ea));
        db = __dadd_rn(db, __dmul_rn(eb, eb));
    }
    const bool half = db < da;
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = half ? b[i] : a[i];
    return half ? 1 : 0;
}

struct In {
    const uint8_t* base;
    int dtype, es;
    int64_t rows, cols, stride, vpr;
    __device__ __forceinline__ double at(int64_t r, int64_t c) const {
        return c < cols ? load_elem(base, dtype, r * stride + c) : 0.0;
    }
};

// ---- row RMS: 32 rows per warp, column order ---------------------------------------------------
constexpr int kRowWarps = 1;  // warps per block of the row kernels (32 rows per block)

__global__ void __launch_bounds__(kRowWarps * 32) rms_kernel(const In in, double* rms, uint32_t* bad) {
    __shared__ double sq[kRowWarps][32][33];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t r0 = (int64_t(blockIdx.x) * kRowWarps + w) * 32;
    if (r0 >= in.rows) return;
    double acc = 0.0;
    bool finite = true;
    for (int64_t c0 = 0; c0 < in.cols; c0 += 32) {
        const int64_t c = c0 + lane;
        double v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)  // all loads first, so their latencies overlap
            v[i] = (r0 + i < in.rows && c < in.cols) ? load_elem(in.base, in.dtype, (r0 + i) * in.stride + c) : 0.0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            finite = finite && isfinite(v[i]);
            sq[w][i][lane] = __dmul_rn(v[i], v[i]);
        }
        __syncwarp();
        const int n = int(in.cols - c0 < 32 ? in.cols - c0 : 32);
        for (int j = 0; j < n; ++j) acc = __dadd_rn(acc, sq[w][lane][j]);
        __syncwarp();
    }
    if (!finite) atomicOr(bad, 1u);
    if (r0 + lane < in.rows) rms[r0 + lane] = __dsqrt_rn(__ddiv_rn(acc, double(in.cols)));
}

// ---- lattice quantisation: one thread per vector -----------------------------------------------
// Rows: all (n_sample == 0) or the sampled rows floor(i * rows / n_sample).  Symbol counts of the
// 16 contexts (field j given coset c at 8c + j - 1) go to counts[16 * 256] and escapes; cosets and
// fields are written when coset != null.
__global__ void __launch_bounds__(256) quant_kernel(const In in, const double* rms, double s, int64_t n_sample,
                                                    unsigned long long* counts, unsigned long long* escapes,
                                                    uint8_t* coset_out, int16_t* fields_out) {
    __shared__ uint32_t hist[16 * 256];
    __shared__ uint32_t esc;
    for (int i = threadIdx.x; i < 16 * 256; i += blockDim.x) hist[i] = 0;
    if (threadIdx.x == 0) esc = 0;
    __syncthreads();
    const int64_t nrows = n_sample ? n_sample : in.rows;
    const int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (g < nrows * in.vpr) {
        const int64_t i = g / in.vpr, k = g - i * in.vpr;
        const int64_t r = n_sample ? (i * in.rows) / n_sample : i;
        const double rr = rms[r];
        double t[8], y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double xh = rr > 0.0 ? __ddiv_rn(in.at(r, 8 * k + e), rr) : 0.0;
            const double v = __ddiv_rn(xh, s);
            t[e] = v > kClampT ? kClampT : (v < -kClampT ? -kClampT : v);
        }
        const int c = nearest_e8(t, y);
        int32_t z[8], f[8], s7 = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) z[e] = int32_t(__dsub_rn(y[e], 0.5 * c));
#pragma unroll
        for (int e = 0; e < 7; ++e) { f[e] = z[e]; s7 += z[e]; }
        f[7] = (z[7] - (s7 & 1)) / 2;
        uint32_t ne = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int sy = symbol_of(f[j]);
            atomicAdd(&hist[256 * (8 * c + j) + sy], 1u);
            ne += sy == kEscape;
        }
        if (ne) atomicAdd(&esc, ne);
        if (coset_out) {
            const int64_t v = r * in.vpr + k;
            coset_out[v] = uint8_t(c);
            int4 pk;
            pk.x = int((uint32_t(uint16_t(f[0]))) | (uint32_t(uint16_t(f[1])) << 16));
            pk.y = int((uint32_t(uint16_t(f[2]))) | (uint32_t(uint16_t(f[3])) << 16));
            pk.z = int((uint32_t(uint16_t(f[4]))) | (uint32_t(uint16_t(f[5])) << 16));
            pk.w = int((uint32_t(uint16_t(f[6]))) | (uint32_t(uint16_t(f[7])) << 16));
            reinterpret_cast<int4*>(fields_out)[v] = pk;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 16 * 256; i += blockDim.x)
        if (hist[i]) atomicAdd(&counts[i], (unsigned long long)hist[i]);
    if (threadIdx.x == 0 && esc) atomicAdd(escapes, (unsigned long long)esc);
}

// ---- row least-squares scales: alpha_r = sum w y / sum y^2 over real columns, column order ----
// Per 32-column chunk of 32 rows (128 vectors), each lane takes 4 vectors: it reads the vector's
// coset and fields once, rebuilds its 8 lattice coordinates (y = z + c/2, z8 = 2 f8 + parity) and
// stages w y and y^2 for every real column; then every lane adds its row's terms in column order.
// The row's largest |2 y| comes from its largest y^2 (exact for half-integers, and so is its root).
__global__ void __launch_bounds__(kRowWarps * 32) alpha_kernel(const In in, const uint8_t* coset,
                                                               const int16_t* fields, float* alpha,
                                                               uint16_t* rowmax) {
    extern __shared__ double sh[];  // [kRowWarps][2][32][33]
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    double (*wy)[33] = reinterpret_cast<double (*)[33]>(sh + size_t(w) * 2 * 32 * 33);
    double (*yy)[33] = reinterpret_cast<double (*)[33]>(sh + size_t(w) * 2 * 32 * 33 + 32 * 33);
    const int64_t r0 = (int64_t(blockIdx.x) * kRowWarps + w) * 32;
    if (r0 >= in.rows) return;
    double swy = 0.0, syy = 0.0, ymax2 = 0.0;
    for (int64_t c0 = 0; c0 < in.cols; c0 += 32) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int q = m * 32 + lane, i = q >> 2, vk = q & 3;
            const int64_t r = r0 + i, col0 = c0 + 8 * vk;
            double a[8], b[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = b[e] = 0.0;
            if (r < in.rows && col0 < in.cols) {
                const int64_t v = r * in.vpr + col0 / 8;
                const int4 pk = reinterpret_cast<const int4*>(fields)[v];
                const int32_t f[8] = {int16_t(pk.x & 0xFFFF), int16_t(uint32_t(pk.x) >> 16),
                                      int16_t(pk.y & 0xFFFF), int16_t(uint32_t(pk.y) >> 16),
                                      int16_t(pk.z & 0xFFFF), int16_t(uint32_t(pk.z) >> 16),
                                      int16_t(pk.w & 0xFFFF), int16_t(uint32_t(pk.w) >> 16)};
                const double half = 0.5 * coset[v];
                const int32_t s7 = f[0] + f[1] + f[2] + f[3] + f[4] + f[5] + f[6];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if (col0 + e < in.cols) {
                        const int32_t z = e < 7 ? f[e] : 2 * f[7] + (s7 & 1);
                        const double y = double(z) + half;  // exact: a half-integer
                        a[e] = __dmul_rn(load_elem(in.base, in.dtype, r * in.stride + col0 + e), y);
                        b[e] = __dmul_rn(y, y);
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                wy[i][8 * vk + e] = a[e];
                yy[i][8 * vk + e] = b[e];
            }
        }
        __syncwarp();
        const int n = int(in.cols - c0 < 32 ? in.cols - c0 : 32);
        for (int j = 0; j < n; ++j) {
            swy = __dadd_rn(swy, wy[lane][j]);
            syy = __dadd_rn(syy, yy[lane][j]);
            ymax2 = fmax(ymax2, yy[lane][j]);
        }
        __syncwarp();
    }
    if (r0 + lane < in.rows) {
        alpha[r0 + lane] = syy > 0.0 ? __double2float_rn(__ddiv_rn(swy, syy)) : 0.0f;
        rowmax[r0 + lane] = uint16_t(2.0 * __dsqrt_rn(ymax2));
    }
}

// ---- rANS tiles: one warp per tile, one lane per state --------------------------------------------
struct TileArgs {
    const uint8_t* coset;
    const int16_t* fields;
    int64_t n_vectors;
    uint32_t steps, n_tiles;
    const uint16_t* q;          // [16][256]
    const uint32_t* cum;        // [16][257]
    uint32_t prob_bits;         // totals M = 2^prob_bits
    uint32_t* lane_words;       // [n_tiles][32]: words of each lane (counting pass output)
    uint64_t* tile_bytes;       // [n_tiles] (counting pass output)
    const uint64_t* tile_off;   // [n_tiles] byte offsets in the stream (writing pass input)
    uint8_t* stream;            // writing pass output (zeroed)
};

constexpr int kTileWarps = 4;

// WRITE = false: count every lane's words and the tile's size.  WRITE = true: write the tile.
template <bool WRITE>
__global__ void __launch_bounds__(kTileWarps * 32) tiles_kernel(const TileArgs a) {
    __shared__ uint16_t q[16][256];
    __shared__ uint32_t cum[16][257];
    for (int i = threadIdx.x; i < 16 * 256; i += blockDim.x) q[i / 256][i % 256] = a.q[i];
    for (int i = threadIdx.x; i < 16 * 257; i += blockDim.x) cum[i / 257][i % 257] = a.cum[i];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const uint32_t tile = blockIdx.x * kTileWarps + (threadIdx.x >> 5);
    if (tile >= a.n_tiles) return;
    const int64_t per_tile = int64_t(kLanes) * a.steps;
    const int64_t v0 = int64_t(tile) * per_tile;
    const int64_t nvec = min(per_tile, a.n_vectors - v0);
    const int64_t steps = (nvec + kLanes - 1) / kLanes;

    // where this lane's words go (writing pass): lane 2p reads its words forward from the region
    // start, lane 2p+1 backward from the region end; emission runs in reverse reading order
    uint8_t* words = nullptr;
    uint32_t n_mine = 0, n_even = 0, region = 0;
    if (WRITE) {
        n_mine = a.lane_words[size_t(tile) * kLanes + lane];
        const uint32_t n_pair = n_mine + __shfl_xor_sync(kFullMask, n_mine, 1);
        n_even = __shfl_sync(kFullMask, n_mine, lane & ~1);
        uint32_t inc = (lane & 1) ? 0u : n_pair;  // one term per pair
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFullMask, inc, o);
            if (lane >= o) inc += t;
        }
        region = __shfl_sync(kFullMask, inc, lane & ~1) - n_pair;  // words before this pair's region
        words = a.stream + a.tile_off[tile] + kTileHeadBytes;
        if (!(lane & 1)) {
            uint8_t* hc = a.stream + a.tile_off[tile] + 4 * kLanes + 2 * (lane >> 1);
            hc[0] = uint8_t(n_pair);
            hc[1] = uint8_t(n_pair >> 8);
        }
    }
    uint32_t emitted = 0;
    auto emit = [&](uint32_t word) {
        if (WRITE) {
            const uint32_t pos = (lane & 1) ? region + n_even + emitted : region + (n_mine - 1 - emitted);
            words[2 * pos] = uint8_t(word);
            words[2 * pos + 1] = uint8_t(word >> 8);
        }
        ++emitted;
    };
    uint32_t x = kStateLow;
    auto code = [&](uint32_t f, uint32_t c) {
        if (uint64_t(x) >= (uint64_t(f) << (32 - a.prob_bits))) {  // renormalise: push 16 bits out
            emit(x & 0xFFFFu);
            x >>= 16;
        }
        x = (x / f) * (1u << a.prob_bits) + (x % f) + c;
    };
    for (int64_t k = steps - 1; k >= 0; --k) {
        const int64_t v = v0 + k * kLanes + lane;
        if (v >= v0 + nvec) continue;
        const int16_t* f = a.fields + 8 * v;
        const int c = a.coset[v];
        for (int j = 7; j >= 0; --j)
            if (symbol_of(f[j]) == kEscape) emit(uint16_t(f[j]));
        for (int j = 7; j >= 1; --j) code(q[8 * c + j][symbol_of(f[j])], cum[8 * c + j][symbol_of(f[j])]);
        const int s1 = symbol_of(f[0]);  // (coset, f1): coset 1's slots follow coset 0's
        code(q[8 * c][s1], cum[8 * c][s1] + (c ? cum[0][256] : 0u));
    }
    if (!WRITE) {
        a.lane_words[size_t(tile) * kLanes + lane] = emitted;
        uint32_t total = emitted;
#pragma unroll
        for (int o = 16; o; o >>= 1) total += __shfl_xor_sync(kFullMask, total, o);
        if (lane == 0) a.tile_bytes[tile] = round_up16(kTileHeadBytes + 2 * uint64_t(total));
    } else {
        uint8_t* st = a.stream + a.tile_off[tile] + 4 * lane;
        st[0] = uint8_t(x);
        st[1] = uint8_t(x >> 8);
        st[2] = uint8_t(x >> 16);
        st[3] = uint8_t(x >> 24);
    }
}

// Device buffers of one encode, from the device's stream-ordered pool (freed memory is reused by
// the next encode without a device-wide synchronisation), released on every exit path.
struct DevBuf {
    cudaStream_t st;
    std::vector<void*> ptrs;
    explicit DevBuf(cudaStream_t s) : st(s) {}
    ~DevBuf() {
        for (void* p : ptrs) cudaFreeAsync(p, st);
    }
    template <class T>
    T* alloc(size_t n) {
        void* p = nullptr;
        if (cudaMallocAsync(&p, std::max<size_t>(n, 1) * sizeof(T), st) != cudaSuccess) return nullptr;
        ptrs.push_back(p);
        return static_cast<T*>(p);
    }
};

}  // namespace

// Encode a device tensor (in.bits is device memory on the current device).  Same result and return
// codes as encode(); -6 for a CUDA failure, -7 for device memory.
int encode_gpu(const EncodeInput& in, double target, const EncodeOptions& opt, std::vector<uint8_t>& blob,
               std::string& why) {
    const int64_t rows = in.rows, cols = in.cols, vpr = (cols + 7) / 8, V = rows * vpr;
    const int S = opt.steps_per_tile > 0 ? opt.steps_per_tile : default_steps(target);
    const int64_t per_tile = int64_t(kLanes) * S;
    const int64_t n_tiles = (V + per_tile - 1) / per_tile;
    if (n_tiles > int64_t(UINT32_MAX) - 1) { why = "too many tiles"; return -3; }
    cudaStream_t st = cudaStreamPerThread;
    DevBuf buf(st);
    auto cuda_fail = [&](cudaError_t e, const char* what) {
        why = std::string(what) + ": " + cudaGetErrorString(e);
        return -6;
    };
#define EPG(call, what)                        \
    do {                                       \
        cudaError_t e_ = (call);               \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

    In d{static_cast<const uint8_t*>(in.bits), in.dtype, dtype_bytes(in.dtype), rows, cols, in.row_stride, vpr};
    double* rms = buf.alloc<double>(size_t(rows));
    uint32_t* bad = buf.alloc<uint32_t>(1);
    unsigned long long* counts = buf.alloc<unsigned long long>(16 * 256 + 1);
    uint8_t* coset = buf.alloc<uint8_t>(size_t(V));
    int16_t* fields = buf.alloc<int16_t>(size_t(V) * 8);
    float* alpha_d = buf.alloc<float>(size_t(rows));
    uint16_t* rowmax_d = buf.alloc<uint16_t>(size_t(rows));
    if (!rms || !bad || !counts || !coset || !fields || !alpha_d || !rowmax_d) { why = "device memory"; return -7; }

    const unsigned row_blocks = unsigned((rows + 32 * kRowWarps - 1) / (32 * kRowWarps));
    EPG(cudaMemsetAsync(bad, 0, 4, st), "encode: clear");
    rms_kernel<<<row_blocks, kRowWarps * 32, 0, st>>>(d, rms, bad);
    EPG(cudaGetLastError(), "encode: row RMS");
    uint32_t bad_h = 0;
    EPG(cudaMemcpyAsync(&bad_h, bad, 4, cudaMemcpyDeviceToHost, st), "encode: read back");
    EPG(cudaStreamSynchronize(st), "encode: row RMS");
    if (bad_h) { why = "input holds a non-finite value"; return -4; }

    // counts of one quantisation pass (all rows or the sample) as host Counts
    std::vector<unsigned long long> ch(16 * 256 + 1);
    auto quantise = [&](double s, int64_t n_sample, bool store, Counts& out) -> int {
        EPG(cudaMemsetAsync(counts, 0, sizeof(unsigned long long) * (16 * 256 + 1), st), "encode: clear");
        const int64_t work = (n_sample ? n_sample : rows) * vpr;
        quant_kernel<<<unsigned((work + 255) / 256), 256, 0, st>>>(d, rms, s, n_sample, counts, counts + 16 * 256,
                                                                    store ? coset : nullptr, store ? fields : nullptr);
        EPG(cudaGetLastError(), "encode: quantise");
        EPG(cudaMemcpyAsync(ch.data(), counts, sizeof(unsigned long long) * ch.size(), cudaMemcpyDeviceToHost, st),
            "encode: read back");
        EPG(cudaStreamSynchronize(st), "encode: quantise");
        for (int i = 0; i < 16 * 256; ++i) out.c[size_t(i)] = ch[size_t(i)];
        out.escapes = ch[16 * 256];
        return 0;
    };

    // Finest scale whose sampled estimate meets the target: bisection on log2 s over [-24, 8].
    const int64_t n_sample = std::min<int64_t>(rows, 256);
    int qrc = 0;
    auto estimate = [&](double s) {
        Counts c;
        qrc = qrc ? qrc : quantise(s, n_sample, false, c);
        return estimate_from_counts(c, rows, cols, n_sample, n_tiles, opt.prob_bits);
    };
    double s;
    if (opt.scale > 0.0) {
        s = opt.scale;
    } else {
        double lo = -24.0, hi = 8.0;
        if (estimate(std::exp2(hi)) > target) s = std::exp2(hi);
        else if (estimate(std::exp2(lo)) <= target) s = std::exp2(lo);
        else {
            for (int it = 0; it < 48; ++it) {
                double mid = 0.5 * (lo + hi);
                if (estimate(std::exp2(mid)) <= target) hi = mid;
                else lo = mid;
            }
            s = std::exp2(hi);
        }
    }
    if (qrc) return qrc;

    // Full quantisation, tables, row scales.
    Counts all;
    if (int rc = quantise(s, 0, true, all)) return rc;
    Tables T;
    T.build(all, opt.prob_bits);
    constexpr size_t kAlphaSmem = size_t(kRowWarps) * 2 * 32 * 33 * sizeof(double);
    EPG(cudaFuncSetAttribute(alpha_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kAlphaSmem)),
        "encode: row scales");
    alpha_kernel<<<row_blocks, kRowWarps * 32, kAlphaSmem, st>>>(d, coset, fields, alpha_d, rowmax_d);
    EPG(cudaGetLastError(), "encode: row scales");
    std::vector<float> alpha(static_cast<size_t>(rows));
    std::vector<uint16_t> rowmax(static_cast<size_t>(rows));
    EPG(cudaMemcpyAsync(alpha.data(), alpha_d, 4 * size_t(rows), cudaMemcpyDeviceToHost, st), "encode: read back");
    EPG(cudaMemcpyAsync(rowmax.data(), rowmax_d, 2 * size_t(rows), cudaMemcpyDeviceToHost, st), "encode: read back");

    // Tiles: count, lay out, write.
    uint16_t* q_d = buf.alloc<uint16_t>(16 * 256);
    uint32_t* cum_d = buf.alloc<uint32_t>(16 * 257);
    uint32_t* lane_words = buf.alloc<uint32_t>(size_t(n_tiles) * kLanes);
    uint64_t* tbytes_d = buf.alloc<uint64_t>(size_t(n_tiles));
    uint64_t* toff_d = buf.alloc<uint64_t>(size_t(n_tiles));
    if (!q_d || !cum_d || !lane_words || !tbytes_d || !toff_d) { why = "device memory"; return -7; }
    EPG(cudaMemcpyAsync(q_d, &T.q[0][0], sizeof T.q, cudaMemcpyHostToDevice, st), "encode: tables");
    EPG(cudaMemcpyAsync(cum_d, &T.cum[0][0], sizeof T.cum, cudaMemcpyHostToDevice, st), "encode: tables");
    TileArgs ta{coset, fields, V, uint32_t(S), uint32_t(n_tiles), q_d, cum_d, uint32_t(T.prob_bits), lane_words,
                tbytes_d, toff_d, nullptr};
    const unsigned tile_blocks = unsigned((n_tiles + kTileWarps - 1) / kTileWarps);
    tiles_kernel<false><<<tile_blocks, kTileWarps * 32, 0, st>>>(ta);
    EPG(cudaGetLastError(), "encode: tile sizes");
    std::vector<uint64_t> tbytes(static_cast<size_t>(n_tiles)), toff(static_cast<size_t>(n_tiles));
    EPG(cudaMemcpyAsync(tbytes.data(), tbytes_d, 8 * size_t(n_tiles), cudaMemcpyDeviceToHost, st), "encode: read back");
    EPG(cudaStreamSynchronize(st), "encode: tile sizes");
    uint64_t stream_bytes = 0;
    for (int64_t t = 0; t < n_tiles; ++t) {
        toff[size_t(t)] = stream_bytes;
        stream_bytes += tbytes[size_t(t)];
    }
    uint64_t off_stream = 0;
    if (!assemble_blob(in.dtype, rows, cols, S, s, T, alpha, rowmax, tbytes, blob, &off_stream, why)) return -3;
    uint8_t* stream_d = buf.alloc<uint8_t>(size_t(stream_bytes));
    if (!stream_d) { why = "device memory"; return -7; }
    EPG(cudaMemsetAsync(stream_d, 0, size_t(stream_bytes), st), "encode: clear");
    EPG(cudaMemcpyAsync(toff_d, toff.data(), 8 * size_t(n_tiles), cudaMemcpyHostToDevice, st), "encode: layout");
    ta.stream = stream_d;
    tiles_kernel<true><<<tile_blocks, kTileWarps * 32, 0, st>>>(ta);
    EPG(cudaGetLastError(), "encode: tiles");
    EPG(cudaMemcpyAsync(blob.data() + off_stream, stream_d, size_t(stream_bytes), cudaMemcpyDeviceToHost, st),
        "encode: read back");
    EPG(cudaStreamSynchronize(st), "encode: tiles");
#undef EPG
    return 0;
}

}  // namespace ep
