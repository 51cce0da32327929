// encoder.cpp -- host encoder of the library (ep_compress).
//
// Steps, as "EntroPack lattice compression" (documentation page) describes them:
//   section "Lattice quantization and integer fields": normalise each row by its RMS, group
//     the normalised values into 8-vectors, replace each by its nearest point of a scaled E8
//     lattice (shared scale s), store the point as a coset bit and eight integer fields with the
//     last coordinate compacted by the parity constraint, model each field conditioned on the
//     coset;
//   section "Rate selection and refinement": choose s from size estimates on sampled rows,
//     then quantise the full tensor and fit one least-squares scale per row;
//   section "Encoding and reconstruction": rANS-code the fields in tiles that decode on their
//     own, and keep the frequency tables, per-row scales and per-tile bookkeeping beside them.
// The rANS coding step is Duda's ("Asymmetric numeral systems", 2009); the E8 nearest point is
// the Conway-Sloane rule (1982).  Details the pages leave open are fixed as the format header
// (format.h) and the comments below state.
//
// Work is split over host threads by rows, sampled rows and tiles; every reduction is over
// integers or in a fixed order, so the bytes do not depend on the thread count.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <functional>
#include <thread>

#include "format.h"
#include "tables.h"

namespace ep {

// ---------------------------------------------------------------------------------------------
// Parallel loop over [0, n) in contiguous blocks.
// ---------------------------------------------------------------------------------------------
static void parallel_for(int64_t n, int threads, const std::function<void(int64_t, int64_t, int)>& body) {
    if (n <= 0) return;
    int T = int(std::max<int64_t>(1, std::min<int64_t>(threads, n)));
    if (T == 1) { body(0, n, 0); return; }
    std::vector<std::thread> pool;
    pool.reserve(T);
    for (int t = 0; t < T; ++t) {
        int64_t a = n * t / T, b = n * (t + 1) / T;
        pool.emplace_back([=, &body] { body(a, b, t); });
    }
    for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------------------------------------
// Reading container elements as exact doubles.
// ---------------------------------------------------------------------------------------------
class ElementReader {
public:
    ElementReader(const void* base, int dtype, int64_t rows, int64_t cols, int64_t stride)
        : base_(static_cast<const uint8_t*>(base)), dtype_(dtype), rows_(rows), cols_(cols), stride_(stride) {
        if (dtype == kFP16) {
            lut_.resize(65536);
            for (uint32_t h = 0; h < 65536; ++h) lut_[h] = half_value(h);
        } else if (dtype == kE4M3) {
            lut_.resize(256);
            for (uint32_t b = 0; b < 256; ++b) lut_[b] = e4m3_value(b);
        }
    }
    // value of (r, c); columns past cols are the zero padding
    double at(int64_t r, int64_t c) const {
        if (c >= cols_) return 0.0;
        size_t idx = size_t(r * stride_ + c);
        switch (dtype_) {
            case kBF16: {
                uint32_t w = uint32_t(reinterpret_cast<const uint16_t*>(base_)[idx]) << 16;
                float f;
                std::memcpy(&f, &w, 4);
                return f;
            }
            case kFP16: return lut_[reinterpret_cast<const uint16_t*>(base_)[idx]];
            case kE4M3: return lut_[base_[idx]];
            case kI8: return double(int8_t(base_[idx]));  // two's complement integer
            default: return reinterpret_cast<const float*>(base_)[idx];
        }
    }

private:
    static double half_value(uint32_t h) {  // IEEE binary16
        int e = (h >> 10) & 0x1F;
        uint32_t m = h & 0x3FF;
        double mag = e == 0 ? std::ldexp(double(m), -24)
                   : e == 31 ? (m ? NAN : INFINITY)
                   : std::ldexp(double(m | 0x400), e - 25);
        return (h & 0x8000) ? -mag : mag;
    }
    static double e4m3_value(uint32_t b) {  // OCP E4M3: bias 7, S.1111.111 is NaN, no inf
        int e = (b >> 3) & 0xF;
        uint32_t m = b & 7;
        double mag = (e == 15 && m == 7) ? NAN
                   : e == 0 ? std::ldexp(double(m), -9)
                   : std::ldexp(double(m | 8), e - 10);
        return (b & 0x80) ? -mag : mag;
    }
    const uint8_t* base_;
    int dtype_;
    int64_t rows_, cols_, stride_;
    std::vector<double> lut_;
};

// ---------------------------------------------------------------------------------------------
// Lattice quantisation.
// ---------------------------------------------------------------------------------------------

// Conway-Sloane nearest point of D8 = {z in Z^8 : sum even}: round every coordinate (halves away
// from zero); on an odd sum move the coordinate that rounding disturbed most (first one on ties)
// one step toward its value (up when it was already an integer).
static inline void nearest_d8(const double u[8], double g[8]) {
    long long sum = 0;
    int worst_i = 0;
    double worst = -1.0;
    for (int i = 0; i < 8; ++i) {
        g[i] = std::round(u[i]);
        sum += (long long)g[i];
        double miss = std::fabs(u[i] - g[i]);
        if (miss > worst) { worst = miss; worst_i = i; }
    }
    if (sum % 2 != 0) g[worst_i] += (u[worst_i] < g[worst_i]) ? -1.0 : 1.0;
}

// Nearest point of E8 = D8 u (D8 + 1/2): the closer of the D8 point and the half-integer coset
// point (the D8 rule on t - 1/2, shifted back); equal distances keep the integer coset.
static inline int nearest_e8(const double t[8], double y[8]) {
    double a[8], b[8], u[8];
    nearest_d8(t, a);
    for (int i = 0; i < 8; ++i) u[i] = t[i] - 0.5;
    nearest_d8(u, b);
    double da = 0.0, db = 0.0;
    for (int i = 0; i < 8; ++i) {
        b[i] += 0.5;
        da += (t[i] - a[i]) * (t[i] - a[i]);
        db += (t[i] - b[i]) * (t[i] - b[i]);
    }
    const double* best = db < da ? b : a;
    for (int i = 0; i < 8; ++i) y[i] = best[i];
    return db < da ? 1 : 0;
}

// One quantised vector: coset bit, eight fields, and the lattice point (in units of s).
struct QVec {
    int coset;
    int32_t f[8];
    double y[8];
};

class Quantiser {
public:
    Quantiser(const ElementReader& rd, int64_t rows, int64_t cols, const std::vector<double>& rms)
        : rd_(rd), rows_(rows), cols_(cols), rms_(rms) {}

    // vector k of row r at shared scale s; |x_hat / s| is clamped to 32764 so that every
    // field fits an int16 raw word.
    void quantise(int64_t r, int64_t k, double s, QVec& q) const {
        double t[8];
        double rr = rms_[size_t(r)];
        for (int i = 0; i < 8; ++i) {
            double xh = rr > 0.0 ? rd_.at(r, 8 * k + i) / rr : 0.0;
            double v = xh / s;
            t[i] = v > 32764.0 ? 32764.0 : (v < -32764.0 ? -32764.0 : v);
        }
        q.coset = nearest_e8(t, q.y);
        // fields: z = y - c/2 in D8; f1..f7 = z1..z7; f8 = (z8 - (z1+...+z7 mod 2)) / 2
        int32_t z[8], s7 = 0;
        for (int i = 0; i < 8; ++i) z[i] = int32_t(q.y[i] - 0.5 * q.coset);
        for (int i = 0; i < 7; ++i) { q.f[i] = z[i]; s7 += z[i]; }
        int32_t par = s7 & 1;
        q.f[7] = (z[7] - par) / 2;
    }

private:
    const ElementReader& rd_;
    int64_t rows_, cols_;
    const std::vector<double>& rms_;
};

// ---------------------------------------------------------------------------------------------
// Tiled, 32-way interleaved rANS.  Lane l of a tile owns vectors l, 32 + l, 64 + l, ... and one
// 32-bit state.  A lane reads its own words: for each step, after each of its 8 decodes ((coset,
// f1) as one symbol, then f2..f8) one word if the state fell below 2^16, then the raw words of its
// escaped fields in field order.  Lanes 2p and 2p+1 share region p: lane 2p reads forward from the region start,
// lane 2p+1 backward from the region end.  Tile: 32 u32 states, 16 u16 region word counts, the
// regions, zero padding to 16 bytes.  Each lane is encoded in reverse reading order.
// ---------------------------------------------------------------------------------------------
static void encode_tile(const uint8_t* coset, const int16_t* fields, int64_t nvec, const Tables& T,
                        std::vector<uint8_t>& out) {
    uint32_t x[kLanes];
    std::vector<uint16_t> lw[kLanes];  // emission order (reverse of reading order)
    const int64_t steps = (nvec + kLanes - 1) / kLanes;
    auto code = [&](uint32_t& st, std::vector<uint16_t>& w, uint32_t f, uint32_t c) {
        if (uint64_t(st) >= (uint64_t(f) << (32 - T.prob_bits))) {  // renormalise: push 16 bits out
            w.push_back(uint16_t(st));
            st >>= 16;
        }
        st = (st / f) * T.M + (st % f) + c;
    };
    auto put = [&](uint32_t& st, std::vector<uint16_t>& w, int ctx, int sym) {
        code(st, w, T.q[ctx][sym], T.cum[ctx][sym]);
    };
    auto put_joint = [&](uint32_t& st, std::vector<uint16_t>& w, int coset, int sym) {
        code(st, w, T.q[8 * coset][sym], T.joint_cum(coset, sym));
    };
    for (int l = 0; l < kLanes; ++l) {
        x[l] = kStateLow;
        lw[l].reserve(size_t(steps) * 5);
        for (int64_t k = steps - 1; k >= 0; --k) {
            const int64_t v = k * kLanes + l;
            if (v >= nvec) continue;
            const int16_t* f = &fields[size_t(8 * v)];
            for (int j = 7; j >= 0; --j)
                if (symbol_of(f[j]) == kEscape) lw[l].push_back(uint16_t(f[j]));
            for (int j = 7; j >= 1; --j) put(x[l], lw[l], 8 * coset[v] + j, symbol_of(f[j]));
            put_joint(x[l], lw[l], coset[v], symbol_of(f[0]));  // (coset, f1): one symbol
        }
    }
    size_t words = 0;
    for (auto& w : lw) words += w.size();
    out.assign(round_up16(kTileHeadBytes + 2 * words), 0);
    for (int l = 0; l < kLanes; ++l) wr32(&out[size_t(4 * l)], x[l]);
    size_t r = kTileHeadBytes;  // byte offset of the current region
    for (int p = 0; p < kPairs; ++p) {
        const auto& fw = lw[2 * p];
        const auto& bw = lw[2 * p + 1];
        const size_t n = fw.size() + bw.size();
        wr16(&out[size_t(4 * kLanes + 2 * p)], uint32_t(n));
        for (size_t i = 0; i < fw.size(); ++i) wr16(&out[r + 2 * i], fw[fw.size() - 1 - i]);
        for (size_t i = 0; i < bw.size(); ++i) wr16(&out[r + 2 * (n - 1 - i)], bw[bw.size() - 1 - i]);
        r += 2 * n;
    }
}

// ---------------------------------------------------------------------------------------------
// The encoder.
// ---------------------------------------------------------------------------------------------
// ---------------------------------------------------------------------------------------------
// Per-row rate-distortion refinement ("EntroPack lattice compression", section "Rate selection
// and refinement": optional, off by default; several resolutions are compared per row and handed
// out under the estimated storage budget, alternating with updates of the shared tables).
// Candidates s * 2^(k/2) for k in {0, -1, 1, -2, 2} (this order breaks ties).  Per candidate:
// D = sum over real columns of (w - alpha y)^2 with alpha the row's fp32 least-squares scale, and
// R = the row's code length under the current tables (log2 M bits for a symbol they do not hold)
// plus 16 bits per escape.  A round picks argmin D + lambda R per row, lambda = 2^u the smallest
// (64 bisection steps on u over [-100, 40]) whose total R meets target * N - 8 * metadata bytes;
// then the tables are rebuilt from the chosen rows.  Three rounds from tables of k = 0.
// ---------------------------------------------------------------------------------------------
constexpr int kRdCandidates = 5, kRdRounds = 3;
constexpr int kRdK[kRdCandidates] = {0, -1, 1, -2, 2};

static double rd_resolution(double s, int ki) { return s * std::exp2(0.5 * kRdK[ki]); }

static std::vector<int> rd_allocate(const ElementReader& rd, const Quantiser& Q, int64_t rows, int64_t cols,
                                    int64_t vpr, double s, double target, int64_t n_tiles, int threads,
                                    int prob_bits) {
    const size_t per = size_t(vpr) * 9, R5 = size_t(kRdCandidates);
    std::vector<uint8_t> sym(size_t(rows) * R5 * per);
    std::vector<uint64_t> nesc(size_t(rows) * R5);
    std::vector<double> D(size_t(rows) * R5), R(size_t(rows) * R5);
    parallel_for(rows, threads, [&](int64_t a, int64_t b, int) {
        QVec q;
        std::vector<double> ys(size_t(vpr) * 8);
        for (int64_t r = a; r < b; ++r)
            for (int ki = 0; ki < kRdCandidates; ++ki) {
                const size_t idx = size_t(r) * R5 + size_t(ki);
                uint8_t* sy = &sym[idx * per];
                uint64_t ne = 0;
                double swy = 0.0, syy = 0.0;
                for (int64_t k = 0; k < vpr; ++k) {
                    Q.quantise(r, k, rd_resolution(s, ki), q);
                    sy[9 * k] = uint8_t(q.coset);
                    for (int j = 0; j < 8; ++j) {
                        sy[9 * k + 1 + j] = uint8_t(symbol_of(q.f[j]));
                        ne += sy[9 * k + 1 + j] == kEscape;
                    }
                    for (int i = 0; i < 8; ++i) {
                        ys[size_t(8 * k + i)] = q.y[i];
                        if (8 * k + i < cols) {
                            swy += rd.at(r, 8 * k + i) * q.y[i];
                            syy += q.y[i] * q.y[i];
                        }
                    }
                }
                const float al = syy > 0.0 ? float(swy / syy) : 0.0f;
                double d = 0.0;
                for (int64_t k = 0; k < vpr; ++k)
                    for (int i = 0; i < 8; ++i)
                        if (8 * k + i < cols) {
                            double e = rd.at(r, 8 * k + i) - double(al) * ys[size_t(8 * k + i)];
                            d += e * e;
                        }
                D[idx] = d;
                nesc[idx] = ne;
            }
    });
    std::vector<int> kr(static_cast<size_t>(rows), 0);
    auto choose = [&](double lambda) {
        double total = 0.0;
        for (int64_t r = 0; r < rows; ++r) {
            const size_t b0 = size_t(r) * R5;
            int best = 0;
            double bc = D[b0] + lambda * R[b0];
            for (int ki = 1; ki < kRdCandidates; ++ki) {
                double c = D[b0 + size_t(ki)] + lambda * R[b0 + size_t(ki)];
                if (c < bc) { bc = c; best = ki; }
            }
            kr[size_t(r)] = best;
            total += R[b0 + size_t(best)];
        }
        return total;
    };
    for (int round = 0; round < kRdRounds; ++round) {
        Counts all;
        for (int64_t r = 0; r < rows; ++r) {
            const uint8_t* sy = &sym[(size_t(r) * R5 + size_t(kr[size_t(r)])) * per];
            for (int64_t k = 0; k < vpr; ++k) {
                const int c = sy[9 * k];
                for (int j = 0; j < 8; ++j) all.c[size_t(256 * (8 * c + j) + sy[9 * k + 1 + j])]++;
            }
        }
        Tables T;
        T.build(all, prob_bits);
        double cost[16 * 256];
        for (int c = 0; c < 16; ++c)
            for (int sy = 0; sy < 256; ++sy)
                cost[256 * c + sy] = T.q[c][sy] ? -std::log2(double(T.q[c][sy]) / double(T.M))
                                                : std::log2(double(T.M));
        parallel_for(rows, threads, [&](int64_t a, int64_t b, int) {
            for (int64_t r = a; r < b; ++r)
                for (int ki = 0; ki < kRdCandidates; ++ki) {
                    const size_t idx = size_t(r) * R5 + size_t(ki);
                    const uint8_t* sy = &sym[idx * per];
                    double bits = 16.0 * double(nesc[idx]);
                    for (int64_t k = 0; k < vpr; ++k) {
                        const int c = sy[9 * k];
                        for (int j = 0; j < 8; ++j) bits += cost[256 * (8 * c + j) + sy[9 * k + 1 + j]];
                    }
                    R[idx] = bits;
                }
        });
        const double meta = metadata_bytes(T, rows, n_tiles);
        const double budget = target * double(rows) * double(cols) - 8.0 * meta;
        if (choose(0.0) > budget) {
            double lo = -100.0, hi = 40.0;
            if (choose(std::exp2(hi)) <= budget) {
                for (int it = 0; it < 64; ++it) {
                    double mid = 0.5 * (lo + hi);
                    if (choose(std::exp2(mid)) <= budget) hi = mid;
                    else lo = mid;
                }
            }
            choose(std::exp2(hi));
        }
    }
    return kr;
}


bool assemble_blob(int dtype, int64_t rows, int64_t cols, int S, double s, const Tables& T,
                   const std::vector<float>& alpha, const std::vector<uint16_t>& rowmax,
                   const std::vector<uint64_t>& tile_bytes, std::vector<uint8_t>& blob, uint64_t* off_stream_out,
                   std::string& why) {
    const int64_t n_tiles = int64_t(tile_bytes.size());
    uint64_t tab = T.section_bytes();
    uint64_t off_tab = kHeaderBytes, off_alpha = off_tab + round_up16(tab);
    uint64_t off_rmax = off_alpha + round_up16(4 * uint64_t(rows));
    uint64_t off_offs = off_rmax + round_up16(2 * uint64_t(rows));
    uint64_t off_stream = off_offs + round_up16(4 * uint64_t(n_tiles + 1));
    uint64_t stream = 0;
    for (uint64_t t : tile_bytes) stream += t;
    if (stream / 16 > UINT32_MAX) { why = "stream exceeds the 64 GiB tile-offset range"; return false; }
    blob.assign(size_t(off_stream + stream), 0);
    uint8_t* p = blob.data();
    std::memcpy(p, "EPK1", 4);
    wr16(p + 4, kVersion);
    p[6] = uint8_t(dtype);
    p[7] = uint8_t(kAlphabetR);
    wr64(p + 8, uint64_t(rows));
    wr64(p + 16, uint64_t(cols));
    wr32(p + 24, uint32_t(S));
    wr32(p + 28, uint32_t(n_tiles));
    std::memcpy(p + 32, &s, 8);
    wr64(p + 40, blob.size());
    wr64(p + 48, off_tab);
    wr64(p + 56, off_alpha);
    wr64(p + 64, off_offs);
    wr64(p + 72, off_stream);
    wr64(p + 80, off_rmax);
    p[88] = uint8_t(T.prob_bits);
    uint8_t* t = p + off_tab;
    for (int c = 0; c < 16; ++c) {
        int lo, cnt;
        T.range(c, lo, cnt);
        wr16(t, T.q[c][kEscape]);
        t[2] = uint8_t(lo);
        t[3] = uint8_t(cnt);
        t += 4;
        for (int i = 0; i < cnt; ++i, t += 2) wr16(t, T.q[c][lo + i]);
    }
    for (int64_t r = 0; r < rows; ++r) {
        uint32_t bitsf;
        std::memcpy(&bitsf, &alpha[size_t(r)], 4);
        wr32(p + off_alpha + 4 * r, bitsf);
        wr16(p + off_rmax + 2 * r, rowmax[size_t(r)]);
    }
    uint64_t acc = 0;
    for (int64_t i = 0; i <= n_tiles; ++i) {
        wr32(p + off_offs + 4 * i, uint32_t(acc / 16));
        if (i < n_tiles) acc += tile_bytes[size_t(i)];
    }
    *off_stream_out = off_stream;
    return true;
}

int encode(const EncodeInput& in, double target, const EncodeOptions& opt, std::vector<uint8_t>& blob,
           std::string& why) {
    const int64_t rows = in.rows, cols = in.cols, vpr = (cols + 7) / 8, V = rows * vpr;
    const int threads = opt.threads > 0 ? opt.threads : std::max(1u, std::thread::hardware_concurrency());
    ElementReader rd(in.bits, in.dtype, rows, cols, in.row_stride);

    // RMS of every row; non-finite weights are rejected.
    std::vector<double> rms(static_cast<size_t>(rows));
    std::atomic<bool> finite{true};
    parallel_for(rows, threads, [&](int64_t a, int64_t b, int) {
        for (int64_t r = a; r < b; ++r) {
            double acc = 0.0;
            for (int64_t c = 0; c < cols; ++c) {
                double v = rd.at(r, c);
                if (!std::isfinite(v)) finite = false;
                acc += v * v;
            }
            rms[size_t(r)] = std::sqrt(acc / double(cols));
        }
    });
    if (!finite) { why = "input holds a non-finite value"; return -4; }
    Quantiser Q(rd, rows, cols, rms);

    const int S = opt.steps_per_tile > 0 ? opt.steps_per_tile : default_steps(target);
    const int64_t per_tile = int64_t(kLanes) * S;
    const int64_t n_tiles = (V + per_tile - 1) / per_tile;
    if (n_tiles > int64_t(UINT32_MAX) - 1) { why = "too many tiles"; return -3; }

    // Size estimate at scale s from min(rows, 256) rows at floor(i * rows / n) (tables.h).
    const int64_t n_sample = std::min<int64_t>(rows, 256);
    auto estimate = [&](double s) {
        std::vector<Counts> part(static_cast<size_t>(threads));
        parallel_for(n_sample, threads, [&](int64_t a, int64_t b, int t) {
            QVec q;
            for (int64_t i = a; i < b; ++i) {
                int64_t r = (i * rows) / n_sample;
                for (int64_t k = 0; k < vpr; ++k) {
                    Q.quantise(r, k, s, q);
                    part[size_t(t)].add(q.coset, q.f);
                }
            }
        });
        Counts all;
        for (auto& p : part) all.merge(p);
        return estimate_from_counts(all, rows, cols, n_sample, n_tiles, opt.prob_bits);
    };

    // Finest scale whose estimate meets the target: bisection on log2 s over [-24, 8].
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

    // Optional per-row resolutions (the rate-distortion refinement).
    std::vector<int> kr;
    if (opt.rd_refine) kr = rd_allocate(rd, Q, rows, cols, vpr, s, target, n_tiles, threads, opt.prob_bits);

    // Full quantisation, least-squares row scales alpha_r = sum w y / sum y^2 (real columns), and
    // each row's largest |2 y| (an integer: y is an integer or a half-integer) over real columns.
    std::vector<uint8_t> coset(static_cast<size_t>(V));
    std::vector<int16_t> fields(static_cast<size_t>(V) * 8);
    std::vector<float> alpha(static_cast<size_t>(rows));
    std::vector<uint16_t> rowmax(static_cast<size_t>(rows));
    std::vector<Counts> part(static_cast<size_t>(threads));
    parallel_for(rows, threads, [&](int64_t a, int64_t b, int t) {
        QVec q;
        for (int64_t r = a; r < b; ++r) {
            double swy = 0.0, syy = 0.0;
            uint32_t m2 = 0;
            const double sr = kr.empty() ? s : rd_resolution(s, kr[size_t(r)]);
            for (int64_t k = 0; k < vpr; ++k) {
                Q.quantise(r, k, sr, q);
                int64_t v = r * vpr + k;
                coset[size_t(v)] = uint8_t(q.coset);
                for (int j = 0; j < 8; ++j) fields[size_t(8 * v + j)] = int16_t(q.f[j]);
                for (int i = 0; i < 8; ++i)
                    if (8 * k + i < cols) {
                        swy += rd.at(r, 8 * k + i) * q.y[i];
                        syy += q.y[i] * q.y[i];
                        m2 = std::max(m2, uint32_t(std::fabs(2.0 * q.y[i])));
                    }
                part[size_t(t)].add(q.coset, q.f);
            }
            alpha[size_t(r)] = syy > 0.0 ? float(swy / syy) : 0.0f;
            rowmax[size_t(r)] = uint16_t(m2);
        }
    });
    Counts all;
    for (auto& p : part) all.merge(p);
    Tables T;
    T.build(all, opt.prob_bits);

    // Tiles.  (A region's word count is a u16: at most 2 * 17 * S words, fine for S <= 1024.)
    std::vector<std::vector<uint8_t>> tiles(static_cast<size_t>(n_tiles));
    parallel_for(n_tiles, threads, [&](int64_t a, int64_t b, int) {
        for (int64_t t = a; t < b; ++t) {
            int64_t v0 = t * per_tile, nv = std::min(per_tile, V - v0);
            encode_tile(&coset[size_t(v0)], &fields[size_t(8 * v0)], nv, T, tiles[size_t(t)]);
        }
    });

    // Serialise.
    std::vector<uint64_t> sizes(static_cast<size_t>(n_tiles));
    for (int64_t i = 0; i < n_tiles; ++i) sizes[size_t(i)] = tiles[size_t(i)].size();
    uint64_t off_stream = 0;
    if (!assemble_blob(in.dtype, rows, cols, S, s, T, alpha, rowmax, sizes, blob, &off_stream, why)) return -3;
    uint64_t acc = 0;
    for (auto& tb : tiles) {
        std::memcpy(blob.data() + off_stream + acc, tb.data(), tb.size());
        acc += tb.size();
    }
    return 0;
}

// ---------------------------------------------------------------------------------------------
// Blob validation.
// ---------------------------------------------------------------------------------------------
bool parse_blob(const uint8_t* d, size_t n, BlobLayout& L, std::string& why) {
    auto fail = [&](const char* m) { why = m; return false; };
    if (n < kHeaderBytes) return fail("shorter than the 96-byte header");
    if (std::memcmp(d, "EPK1", 4) != 0) return fail("bad magic");
    if (rd16(d + 4) != kVersion) return fail("unknown version");
    L.dtype = d[6];
    if (dtype_bytes(L.dtype) == 0) return fail("unknown dtype");
    if (d[7] != kAlphabetR) return fail("unsupported alphabet");
    L.rows = int64_t(rd64(d + 8));
    L.cols = int64_t(rd64(d + 16));
    L.steps = rd32(d + 24);
    L.n_tiles = rd32(d + 28);
    std::memcpy(&L.scale, d + 32, 8);
    L.total = rd64(d + 40);
    L.off_tables = rd64(d + 48);
    L.off_alpha = rd64(d + 56);
    L.off_offsets = rd64(d + 64);
    L.off_stream = rd64(d + 72);
    L.off_rowmax = rd64(d + 80);
    L.prob_bits = d[88];
    if (!prob_bits_ok(L.prob_bits)) return fail("frequency total is neither 10 nor 12 bits");
    const uint32_t M = 1u << L.prob_bits;
    if (L.total != n) return fail("stored size differs from the byte count");
    if (L.rows <= 0 || L.cols <= 0 || L.rows > (int64_t(1) << 40) || L.cols > (int64_t(1) << 33))
        return fail("bad shape");  // (the decoder keeps a row's vector index in 32 bits)
    if (L.steps == 0 || L.steps > 1024) return fail("bad steps per tile");
    L.vec_per_row = (L.cols + 7) / 8;
    L.n_vectors = L.rows * L.vec_per_row;
    int64_t per = int64_t(kLanes) * L.steps;
    if (int64_t(L.n_tiles) != (L.n_vectors + per - 1) / per) return fail("tile count does not match the shape");
    auto aligned = [](uint64_t o) { return (o & 15) == 0; };
    if (!aligned(L.off_tables) || !aligned(L.off_alpha) || !aligned(L.off_rowmax) || !aligned(L.off_offsets) ||
        !aligned(L.off_stream))
        return fail("misaligned section");
    if (L.off_tables < kHeaderBytes || L.off_tables > L.off_alpha ||
        L.off_alpha + 4 * uint64_t(L.rows) > L.off_rowmax || L.off_rowmax + 2 * uint64_t(L.rows) > L.off_offsets ||
        L.off_offsets + 4 * (uint64_t(L.n_tiles) + 1) > L.off_stream || L.off_stream > n)
        return fail("sections overlap or run past the end");
    uint64_t pos = L.off_tables;
    uint32_t sums[kFieldContexts];
    for (int c = 0; c < kFieldContexts; ++c) {
        if (pos + 4 > L.off_alpha) return fail("table section truncated");
        L.esc_q[c] = rd16(d + pos);
        L.lo[c] = d[pos + 2];
        L.n[c] = d[pos + 3];
        if (int(L.lo[c]) + L.n[c] > kEscape) return fail("table symbol range past 254");
        L.q_offset[c] = uint32_t(pos + 4);
        pos += 4 + 2 * uint64_t(L.n[c]);
        if (pos > L.off_alpha) return fail("table section truncated");
        uint32_t sum = L.esc_q[c];
        for (int i = 0; i < L.n[c]; ++i) sum += rd16(d + L.q_offset[c] + 2 * i);
        sums[c] = sum;
        if (c != 0 && c != 8 && sum != 0 && sum != M) return fail("field table does not sum to its total");
    }
    L.joint_split = sums[0];  // coset-0 half of the joint (coset, f1) table
    if (sums[0] + sums[8] != M) return fail("joint (coset, f1) table does not sum to its total");
    for (int c = 0; c < kFieldContexts; ++c)
        if (L.esc_q[c]) L.has_escape = 1;
    const uint8_t* off = d + L.off_offsets;
    uint64_t stream = n - L.off_stream, prev = 0;
    if (rd32(off) != 0) return fail("first tile offset is not 0");
    for (uint64_t i = 1; i <= L.n_tiles; ++i) {
        uint64_t o = uint64_t(rd32(off + 4 * i)) * 16;
        if (o < prev + kTileHeadBytes) return fail("tile shorter than its 160-byte header");
        L.max_tile_bytes = std::max<uint64_t>(L.max_tile_bytes, o - prev);
        prev = o;
    }
    if (prev != stream) return fail("tile offsets do not end at the stream end");
    return true;
}

}  // namespace ep
