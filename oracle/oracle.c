/*
 * oracle.c -- reference implementation (the oracle) of the EntroPack-style lattice-rANS
 * weight codec: encoder, blob writer and decoder.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark load this library.  The product path (the CUDA library and its host encoder) never
 * calls it, and the two share no code, header, table or constant.
 *
 * Plain, single-threaded C99 in double precision, written to be checked by eye against the
 * method's description rather than to be fast.  Sources, cited by page title and section:
 *
 *   [ABS]  "EntroPack: Fast and Accurate Entropy-Coded Weight Compression at Arbitrary
 *          Bitrates", arXiv abstract page (row-normalised E8 quantisation, conditional model,
 *          sampled storage estimates, tiles that decode on their own, BF16/FP16/FP8/INT8
 *          containers).
 *   [DOC]  "EntroPack lattice compression", documentation page Principles / Lattice-rANS:
 *            DOC-0  opening paragraph (2-D tensors; any finite rate from 0.001 to 11 bits
 *                   per element; the restored tensor has the input's element type);
 *            DOC-LQ section "Lattice quantization and integer fields";
 *            DOC-RS section "Rate selection and refinement";
 *            DOC-ER section "Encoding and reconstruction";
 *            DOC-U  section "Usage".
 *   [ANS]  J. Duda, "Asymmetric numeral systems" (2009) -- the rANS coding step; cited in the
 *          reference list of the Crossref record "Learned Lossless Image Compression with
 *          Interleaved Parallel Inference and Irregular Causal Reasoning".
 *   [CS]   J. H. Conway and N. J. A. Sloane, "Fast quantizing and decoding algorithms for lattice
 *          quantizers and codes" (1982): nearest point of D8, and of E8 = D8 u (D8 + 1/2).
 *   [OCP]  OCP 8-bit floating point specification: the E4M3 encoding (bias 7, no infinities,
 *          largest finite 448).
 *
 * Where the pages leave a step open, the step is marked "reading:" and the same reading is
 * listed in the design notes.  The format these functions write and read is the blob format
 * described there; it is restated next to each writer below.
 *
 * Parity status of each function (which independent check pins it) is listed in the test
 * suite's oracle pin file; every function here is pinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* Constants of the format.                                                                    */
/* ------------------------------------------------------------------------------------------ */

enum { ORC_BF16 = 1, ORC_FP16 = 2, ORC_E4M3 = 3, ORC_F32 = 4, ORC_INT8 = 5 };

#define ORC_R 127          /* reading: field alphabet [-R, R] coded directly, R = 127     */
#define ORC_ESC 255        /* symbol that announces a raw 16-bit field value               */
#define ORC_PB_DEFAULT 12  /* frequency totals: 12-bit (M = 4096), the fixed format choice */
#define ORC_M_MAX 4096u    /* largest total M = 2^prob_bits; prob_bits is 12 or 10         */
#define ORC_L 65536u       /* rANS lower bound 2^16, 32-bit state, 16-bit renormalisation */
#define ORC_VERSION 4      /* blob format version (4: totals in the header, row maxima)   */
#define ORC_LANES 32       /* interleaved rANS states per tile                            */
#define ORC_NCTX 16        /* field j given coset c: 8c + (j-1); 0 and 8 = joint (c, f1)  */
#define ORC_HEADER 96      /* bytes in the fixed header                                   */
#define ORC_CLAMP 32764.0  /* reading: |t| clamp, keeps every field inside int16          */

/* ------------------------------------------------------------------------------------------ */
/* Little-endian byte access.                                                                  */
/* ------------------------------------------------------------------------------------------ */

static void put16(uint8_t* p, uint32_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put32(uint8_t* p, uint32_t v) { for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i)); }
static void put64(uint8_t* p, uint64_t v) { for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i)); }
static uint32_t get16(const uint8_t* p) { return (uint32_t)p[0] | ((uint32_t)p[1] << 8); }
static uint32_t get32(const uint8_t* p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t get64(const uint8_t* p) {
    uint64_t v = 0;
    for (int i = 7; i >= 0; i--) v = (v << 8) | p[i];
    return v;
}
static uint64_t pad16(uint64_t n) { return (n + 15u) / 16u * 16u; }

/* ------------------------------------------------------------------------------------------ */
/* Number formats: reading each container exactly, and rounding to it.                        */
/* [DOC-0]: the tensor is restored in the input's dtype; [ABS] lists BF16, FP16, FP8 and INT8. */
/* ------------------------------------------------------------------------------------------ */

/* Exact value of one stored element of the given dtype. */
double orc_dtype_to_f64(uint32_t bits, int dtype)
{
    if (dtype == ORC_BF16) {                       /* BF16 = the high half of an fp32 */
        uint32_t w = bits << 16;
        float f;
        memcpy(&f, &w, 4);
        return (double)f;
    }
    if (dtype == ORC_F32) {
        float f;
        memcpy(&f, &bits, 4);
        return (double)f;
    }
    if (dtype == ORC_FP16) {                       /* IEEE binary16: 1 + 5 + 10 bits */
        int s = (bits >> 15) & 1, e = (bits >> 10) & 31, m = bits & 1023;
        double v;
        if (e == 0) v = ldexp((double)m, -24);
        else if (e == 31) v = m ? NAN : INFINITY;
        else v = ldexp((double)(1024 + m), e - 25);
        return s ? -v : v;
    }
    if (dtype == ORC_E4M3) {                       /* [OCP] E4M3: 1 + 4 + 3 bits, bias 7 */
        int s = (bits >> 7) & 1, e = (bits >> 3) & 15, m = bits & 7;
        double v;
        if (e == 15 && m == 7) v = NAN;
        else if (e == 0) v = ldexp((double)m, -9);
        else v = ldexp((double)(8 + m), e - 10);
        return s ? -v : v;
    }
    if (dtype == ORC_INT8) return (double)(int8_t)(uint8_t)bits;   /* two's complement */
    return NAN;
}

/*
 * Round v to a binary format with p significand bits, smallest normal exponent emin and largest
 * finite value maxf, ties to even.  v must be finite.  The quantum (the value of the last
 * significand bit) is 2^(max(exponent(v), emin) - (p - 1)); v / quantum is exact because the
 * quantum is a power of two, and rint() rounds it half-to-even in the default rounding mode.
 */
static double round_to_format(double v, int p, int emin, double maxf, int* overflow)
{
    *overflow = 0;
    if (v == 0.0) return v;
    int e;
    frexp(v, &e);                                  /* v = m * 2^e with 0.5 <= |m| < 1 */
    int lead = e - 1;                              /* exponent of the leading bit     */
    if (lead < emin) lead = emin;                  /* subnormal range: fixed quantum  */
    double quantum = ldexp(1.0, lead - (p - 1));
    double r = rint(v / quantum) * quantum;
    if (fabs(r) > maxf) *overflow = 1;
    return r;
}

/* fp32 with round-to-nearest-even; returns the fp32 bit pattern. */
uint32_t orc_round_f32(double v)
{
    uint32_t bits;
    float f;
    if (isnan(v)) { bits = 0x7FC00000u; return bits; }
    if (isinf(v)) { f = (float)v; memcpy(&bits, &f, 4); return bits; }
    int ovf;
    double r = round_to_format(v, 24, -126, (double)3.4028234663852886e38, &ovf);
    if (ovf) r = r > 0 ? INFINITY : -INFINITY;
    f = (float)r;                                  /* exact: r is an fp32 value */
    memcpy(&bits, &f, 4);
    return bits;
}

/* fp32 bit pattern -> BF16 (8 significand bits, fp32 exponent range), RNE, overflow -> inf. */
uint32_t orc_f32_to_bf16(uint32_t fbits)
{
    float f;
    memcpy(&f, &fbits, 4);
    uint32_t sign = (fbits >> 16) & 0x8000u;
    if (isnan(f)) return sign | 0x7FC0u;
    if (isinf(f)) return sign | 0x7F80u;
    int ovf;
    double r = round_to_format((double)f, 8, -126, ldexp(255.0, 120), &ovf);
    if (ovf) return sign | 0x7F80u;
    float g = (float)r;                            /* exact: r has 8 significant bits */
    uint32_t gb;
    memcpy(&gb, &g, 4);
    return (gb >> 16) | sign;                      /* keeps the sign of a zero too */
}

/* fp32 bit pattern -> IEEE binary16, RNE with subnormals, overflow -> inf. */
uint32_t orc_f32_to_f16(uint32_t fbits)
{
    float f;
    memcpy(&f, &fbits, 4);
    uint32_t sign = (fbits >> 16) & 0x8000u;
    if (isnan(f)) return sign | 0x7E00u;
    if (isinf(f)) return sign | 0x7C00u;
    int ovf;
    double r = fabs(round_to_format((double)f, 11, -14, 65504.0, &ovf));
    if (ovf) return sign | 0x7C00u;
    if (r < ldexp(1.0, -14)) return sign | (uint32_t)(r / ldexp(1.0, -24));   /* subnormal or 0 */
    int e;
    frexp(r, &e);
    int lead = e - 1;                              /* -14 .. 15 */
    uint32_t mant = (uint32_t)(r / ldexp(1.0, lead - 10)) - 1024u;
    return sign | ((uint32_t)(lead + 15) << 10) | mant;
}

/* fp32 bit pattern -> OCP E4M3, RNE, saturating to +-448 (no infinities); NaN -> NaN. */
uint32_t orc_f32_to_e4m3(uint32_t fbits)
{
    float f;
    memcpy(&f, &fbits, 4);
    uint32_t sign = (fbits >> 24) & 0x80u;
    if (isnan(f)) return sign | 0x7Fu;
    if (isinf(f)) return sign | 0x7Eu;            /* saturate */
    int ovf;
    double r = fabs(round_to_format((double)f, 4, -6, 448.0, &ovf));
    if (ovf) return sign | 0x7Eu;                 /* saturate */
    if (r < ldexp(1.0, -6)) return sign | (uint32_t)(r / ldexp(1.0, -9));     /* subnormal or 0 */
    int e;
    frexp(r, &e);
    int lead = e - 1;                              /* -6 .. 8 */
    uint32_t mant = (uint32_t)(r / ldexp(1.0, lead - 3)) - 8u;
    return sign | ((uint32_t)(lead + 7) << 3) | mant;
}

/* fp32 bit pattern -> INT8.  reading: the integer container takes the nearest integer, ties to
 * even (the rounding the float containers use), saturating to [-128, 127] as E4M3 saturates;
 * NaN, which no reconstruction produces, gives 0.  rint() rounds half-to-even in the default
 * rounding mode. */
uint32_t orc_f32_to_i8(uint32_t fbits)
{
    float f;
    memcpy(&f, &fbits, 4);
    if (isnan(f)) return 0;
    double r = rint((double)f);
    if (r > 127.0) r = 127.0;
    if (r < -128.0) r = -128.0;
    return (uint32_t)(uint8_t)(int8_t)r;
}

/* Array form of the conversions (used by the exhaustive conversion checks). */
void orc_cvt_f32_array(const uint32_t* in, uint64_t n, int dtype_out, void* out)
{
    for (uint64_t i = 0; i < n; i++) {
        if (dtype_out == ORC_BF16) ((uint16_t*)out)[i] = (uint16_t)orc_f32_to_bf16(in[i]);
        else if (dtype_out == ORC_FP16) ((uint16_t*)out)[i] = (uint16_t)orc_f32_to_f16(in[i]);
        else if (dtype_out == ORC_E4M3) ((uint8_t*)out)[i] = (uint8_t)orc_f32_to_e4m3(in[i]);
        else if (dtype_out == ORC_INT8) ((uint8_t*)out)[i] = (uint8_t)orc_f32_to_i8(in[i]);
        else ((uint32_t*)out)[i] = in[i];
    }
}

/* Store one reconstructed value w (exact, double) into out[idx] of dtype dtype_out:
 * first the fp32 product rounding, then the container rounding. */
static void store_value(void* out, uint64_t idx, int dtype_out, double w)
{
    uint32_t fb = orc_round_f32(w);
    if (dtype_out == ORC_BF16) ((uint16_t*)out)[idx] = (uint16_t)orc_f32_to_bf16(fb);
    else if (dtype_out == ORC_FP16) ((uint16_t*)out)[idx] = (uint16_t)orc_f32_to_f16(fb);
    else if (dtype_out == ORC_E4M3) ((uint8_t*)out)[idx] = (uint8_t)orc_f32_to_e4m3(fb);
    else if (dtype_out == ORC_INT8) ((uint8_t*)out)[idx] = (uint8_t)orc_f32_to_i8(fb);
    else ((uint32_t*)out)[idx] = fb;
}

static int dtype_size(int dtype)
{
    return (dtype == ORC_E4M3 || dtype == ORC_INT8) ? 1 : dtype == ORC_F32 ? 4
           : (dtype == ORC_BF16 || dtype == ORC_FP16) ? 2 : 0;
}

static uint32_t load_bits(const void* data, int dtype, uint64_t i)
{
    if (dtype == ORC_E4M3 || dtype == ORC_INT8) return ((const uint8_t*)data)[i];
    if (dtype == ORC_F32) return ((const uint32_t*)data)[i];
    return ((const uint16_t*)data)[i];
}

/* ------------------------------------------------------------------------------------------ */
/* E8 nearest point [CS], used as [DOC-LQ] describes: nearest point of a scaled E8.            */
/* ------------------------------------------------------------------------------------------ */

/*
 * Nearest point of D8 = { z in Z^8 : sum z even } to u [CS]: round every coordinate to the
 * nearest integer; if the sum of the rounded vector is odd, round the coordinate that was
 * furthest from its integer the other way.
 * reading: ties in rounding go away from zero (C round()); ties for the furthest coordinate go
 * to the lowest index; when that coordinate is exactly an integer, "the other way" is +1.
 */
static void d8_nearest(const double u[8], double g[8])
{
    long long sum = 0;
    for (int i = 0; i < 8; i++) {
        g[i] = round(u[i]);
        sum += (long long)g[i];
    }
    if (sum % 2 != 0) {
        int k = 0;
        double worst = -1.0;
        for (int i = 0; i < 8; i++) {
            double d = fabs(u[i] - g[i]);
            if (d > worst) { worst = d; k = i; }
        }
        if (u[k] > g[k]) g[k] += 1.0;
        else if (u[k] < g[k]) g[k] -= 1.0;
        else g[k] += 1.0;
    }
}

/*
 * Nearest point of E8 = D8 u (D8 + 1/2) to t [CS]: take the nearest point of D8 and the nearest
 * point of the half-integer coset (the D8 rule applied to t - 1/2, then + 1/2), and keep the
 * nearer of the two.  The coset bit is 0 for the integer coset and 1 for the half-integer one
 * ([DOC-LQ]: the two cosets of E8 are its all-integer and all-half-integer points).
 * reading: an exact tie in squared distance keeps coset 0.
 */
void orc_e8_nearest(const double t[8], double y[8], int* coset)
{
    double a[8], b[8], u[8];
    d8_nearest(t, a);
    for (int i = 0; i < 8; i++) u[i] = t[i] - 0.5;
    d8_nearest(u, b);
    for (int i = 0; i < 8; i++) b[i] += 0.5;
    double da = 0.0, db = 0.0;
    for (int i = 0; i < 8; i++) {
        da += (t[i] - a[i]) * (t[i] - a[i]);
        db += (t[i] - b[i]) * (t[i] - b[i]);
    }
    if (db < da) {
        memcpy(y, b, sizeof b);
        *coset = 1;
    } else {
        memcpy(y, a, sizeof a);
        *coset = 0;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Coset bit + eight integer fields [DOC-LQ].                                                 */
/* ------------------------------------------------------------------------------------------ */

/*
 * Lattice point -> fields.  z = y - c/2 lies in D8 (sum even).  f1..f7 = z1..z7, and the
 * parity constraint compacts the last coordinate: with par = (z1 + ... + z7) mod 2 in {0, 1},
 * z8 - par is even and f8 = (z8 - par) / 2 ([DOC-LQ]: E8's even-sum rule lets the last
 * coordinate be stored at half size).
 * reading: for coset 1 the half is subtracted (z = y - 1/2).
 */
void orc_point_to_fields(const double y[8], int coset, int32_t f[8])
{
    int32_t z[8];
    for (int i = 0; i < 8; i++) z[i] = (int32_t)(y[i] - 0.5 * coset);
    int32_t s7 = 0;
    for (int i = 0; i < 7; i++) s7 += z[i];
    int32_t par = ((s7 % 2) + 2) % 2;
    for (int i = 0; i < 7; i++) f[i] = z[i];
    f[7] = (z[7] - par) / 2;
}

/* Fields -> lattice point by arithmetic alone, no table of points ([DOC-LQ]: the fields are
 * invertible): z8 = 2 f8 + par, y = z + c/2. */
void orc_fields_to_point(int coset, const int32_t f[8], double y[8])
{
    int32_t z[8];
    int32_t s7 = 0;
    for (int i = 0; i < 7; i++) { z[i] = f[i]; s7 += f[i]; }
    int32_t par = ((s7 % 2) + 2) % 2;
    z[7] = 2 * f[7] + par;
    for (int i = 0; i < 8; i++) y[i] = (double)z[i] + 0.5 * coset;
}

/* Field value -> symbol of the 256-letter alphabet.  reading: |f| <= 127 is coded as f + 127
 * (symbols 0..254); anything else is the escape symbol 255 followed by the raw 16-bit value. */
static int field_symbol(int32_t f) { return (f >= -ORC_R && f <= ORC_R) ? f + ORC_R : ORC_ESC; }

/* ------------------------------------------------------------------------------------------ */
/* Probability tables with totals M = 2^prob_bits: 4096 (12-bit, the fixed choice) or 1024.    */
/* ------------------------------------------------------------------------------------------ */

/*
 * Quantise symbol counts n[0..nb-1] to frequencies q[] summing to M.
 * reading: q_s = max(1, round_half_up(M n_s / N)) for n_s > 0, else 0; then, while the sum
 * exceeds M, decrement the largest q (> 1; lowest symbol on ties); while it is below M,
 * increment the symbol with the largest count (lowest symbol on ties).  N = 0 gives all zeros.
 */
static void quantize_n(const uint64_t* n, int nb, uint16_t* q, uint32_t M)
{
    uint64_t N = 0;
    for (int s = 0; s < nb; s++) N += n[s];
    for (int s = 0; s < nb; s++) q[s] = 0;
    if (N == 0) return;
    long sum = 0;
    for (int s = 0; s < nb; s++) {
        if (n[s] == 0) continue;
        uint64_t v = (2u * (uint64_t)M * n[s] + N) / (2u * N);  /* round half up */
        if (v < 1) v = 1;
        q[s] = (uint16_t)v;
        sum += (long)v;
    }
    while (sum > (long)M) {
        int best = -1;
        for (int s = 0; s < nb; s++)
            if (q[s] > 1 && (best < 0 || q[s] > q[best])) best = s;
        q[best]--;
        sum--;
    }
    while (sum < (long)M) {
        int best = -1;
        for (int s = 0; s < nb; s++)
            if (n[s] > 0 && (best < 0 || n[s] > n[best])) best = s;
        q[best]++;
        sum++;
    }
}

void orc_quantize_table(const uint64_t n[256], uint16_t q[256], int prob_bits)
{
    quantize_n(n, 256, q, 1u << prob_bits);
}

/*
 * The 16 context tables from symbol counts cnt[16 x 256].  reading: the coset and the first field
 * are one symbol ([DOC-LQ]: every field is modelled given the coset; coding the pair (c, f1) as
 * one symbol of the joint distribution P(c) P(f1 | c) keeps that model and spends one rANS step
 * where two would do): contexts 0 and 8 are the two coset halves of one 512-symbol table,
 * quantised together to sum to M (coset-major order, so ties go to coset 0 first); every other
 * context (c, j >= 2) is quantised on its own.
 */
static void build_tables16(const uint64_t* cnt, uint16_t* q16, int prob_bits)
{
    uint64_t nj[512];
    uint16_t qj[512];
    memcpy(nj, cnt, 256 * sizeof(uint64_t));
    memcpy(nj + 256, cnt + 256 * 8, 256 * sizeof(uint64_t));
    quantize_n(nj, 512, qj, 1u << prob_bits);
    memcpy(q16, qj, 256 * sizeof(uint16_t));
    memcpy(q16 + 256 * 8, qj + 256, 256 * sizeof(uint16_t));
    for (int ctx = 1; ctx < ORC_NCTX; ctx++)
        if (ctx != 8) orc_quantize_table(cnt + 256 * ctx, q16 + 256 * ctx, prob_bits);
}

/* Exposed for the table checks. */
void orc_build_tables16(const uint64_t* cnt, uint16_t* q16, int prob_bits) { build_tables16(cnt, q16, prob_bits); }

/* Cumulative frequencies: cum[s] = q[0] + ... + q[s-1]. */
static void cumulate(const uint16_t q[256], uint32_t cum[257])
{
    cum[0] = 0;
    for (int s = 0; s < 256; s++) cum[s + 1] = cum[s] + q[s];
}

/* Context of field j (1..8) of a vector with coset c. */
static int context_of(int j, int c) { return 8 * c + (j - 1); }

/* Frequency and cumulative frequency of symbol s of field j given coset c.  For j = 1 the two
 * coset halves (contexts 0 and 8) are one distribution over (c, s): coset 1's slots follow all
 * of coset 0's. */
static void freq_cum(const uint16_t* q16, const uint32_t cum[ORC_NCTX][257], int j, int c, int s,
                     uint32_t* q, uint32_t* cm)
{
    int ctx = context_of(j, c);
    *q = q16[256 * ctx + s];
    *cm = cum[ctx][s] + ((j == 1 && c == 1) ? cum[0][256] : 0u);
}

/* ------------------------------------------------------------------------------------------ */
/* Tiled, 32-way interleaved rANS [ANS] with the word layout of the format ([DOC-ER]: the      */
/* fields are rANS-coded in tiles, each of which decodes without the others).                  */
/*                                                                                            */
/* One tile holds up to 32*S consecutive vectors; lane l at step k owns vector 32k + l of the  */
/* tile and has its own 32-bit rANS state.  Each vector is 8 symbols: (coset, f1) jointly, then */
/* f2..f8 (context 8c + j - 1).  A lane's words, in the order it reads them: for each step, for */
/* each of the 8 symbols, after decoding it, one 16-bit word if the state fell below 2^16;     */
/* after the last the raw words of its escaped fields, by field.                               */
/* reading: lanes 2p and 2p+1 share region p: lane 2p's words run forward from the region's    */
/* start, lane 2p+1's run backward from its end.                                                */
/* Tile bytes: 32 little-endian u32 initial states (lane order); 16 u16 word counts of the      */
/* regions (pairs); the regions in pair order; zero padding to a multiple of 16 bytes.  Every  */
/* lane ends in state 2^16, and in every region the two lanes' words meet exactly.             */
/* ------------------------------------------------------------------------------------------ */

#define ORC_PAIRS (ORC_LANES / 2)
#define ORC_TILE_HEAD (4 * ORC_LANES + 2 * ORC_PAIRS)   /* 160 bytes: states + region counts */

typedef struct {
    uint16_t* w;
    uint64_t n, cap;
} wordbuf;

static int push_word(wordbuf* b, uint32_t v)
{
    if (b->n == b->cap) {
        uint64_t nc = b->cap ? 2 * b->cap : 64;
        uint16_t* nw = (uint16_t*)realloc(b->w, nc * sizeof(uint16_t));
        if (!nw) return -1;
        b->w = nw;
        b->cap = nc;
    }
    b->w[b->n++] = (uint16_t)v;
    return 0;
}

/*
 * Encode one tile.  sym9[v*9] is the coset of vector v and sym9[v*9 + j] the symbol of its field j,
 * raw8[v*8 + j-1] the raw value of field j (used when its symbol is the escape).  q16 holds the 16
 * context tables (16 x 256 frequencies summing to M = 2^prob_bits; contexts 0 and 8 the joint
 * (coset, f1) table).  Returns the tile size in bytes (written to out when out != NULL and cap is
 * large enough), or 0 on failure.
 *
 * rANS encode of symbol s with frequency q and cumulative cum [ANS]: while x >= q * (L / M) * 2^16
 * (= q * 2^(32 - prob_bits)), emit the low 16 bits of x and shift them out; then
 * x <- floor(x / q) * M + (x mod q) + cum.
 * Each lane is encoded on its own, in reverse of its reading order, and its words are reversed
 * at the end.
 */
uint64_t orc_encode_tile(const uint8_t* sym9, const int16_t* raw8, int64_t nvec,
                         const uint16_t* q16, int prob_bits, uint8_t* out, uint64_t cap)
{
    const uint32_t M = 1u << prob_bits;
    uint32_t cum[ORC_NCTX][257];
    for (int c = 0; c < ORC_NCTX; c++) cumulate(q16 + 256 * c, cum[c]);
    uint32_t x[ORC_LANES];
    wordbuf wb[ORC_LANES];
    memset(wb, 0, sizeof wb);
    int64_t nsteps = (nvec + ORC_LANES - 1) / ORC_LANES;
    uint64_t bytes = 0;
    for (int l = 0; l < ORC_LANES; l++) {
        x[l] = ORC_L;
        for (int64_t k = nsteps - 1; k >= 0; k--) {
            int64_t v = k * ORC_LANES + l;
            if (v >= nvec) continue;
            for (int j = 8; j >= 1; j--)
                if (sym9[v * 9 + j] == ORC_ESC)
                    if (push_word(&wb[l], (uint16_t)raw8[v * 8 + (j - 1)])) goto fail;
            for (int j = 8; j >= 1; j--) {      /* j = 1 codes the coset too */
                uint32_t q, cm;
                freq_cum(q16, cum, j, sym9[v * 9], sym9[v * 9 + j], &q, &cm);
                if (q == 0) goto fail;
                if ((uint64_t)x[l] >= (uint64_t)q * (ORC_L / M) * 65536u) {
                    if (push_word(&wb[l], x[l] & 0xFFFFu)) goto fail;
                    x[l] >>= 16;
                }
                x[l] = (x[l] / q) * M + (x[l] % q) + cm;
            }
        }
    }
    {
        uint64_t words = 0;
        for (int l = 0; l < ORC_LANES; l++) words += wb[l].n;
        for (int p = 0; p < ORC_PAIRS; p++)
            if (wb[2 * p].n + wb[2 * p + 1].n > 0xFFFFu) goto fail;
        bytes = pad16(ORC_TILE_HEAD + 2u * words);
        if (out && cap >= bytes) {
            memset(out, 0, bytes);
            for (int l = 0; l < ORC_LANES; l++) put32(out + 4 * l, x[l]);
            uint8_t* r = out + ORC_TILE_HEAD;
            for (int p = 0; p < ORC_PAIRS; p++) {
                const wordbuf* e = &wb[2 * p];       /* forward lane */
                const wordbuf* o = &wb[2 * p + 1];   /* backward lane */
                uint64_t n = e->n + o->n;
                put16(out + 4 * ORC_LANES + 2 * p, (uint32_t)n);
                /* reading order is the reverse of emission order */
                for (uint64_t i = 0; i < e->n; i++) put16(r + 2 * i, e->w[e->n - 1 - i]);
                for (uint64_t i = 0; i < o->n; i++) put16(r + 2 * (n - 1 - i), o->w[o->n - 1 - i]);
                r += 2 * n;
            }
        }
    }
    for (int l = 0; l < ORC_LANES; l++) free(wb[l].w);
    return bytes;
fail:
    for (int l = 0; l < ORC_LANES; l++) free(wb[l].w);
    return 0;
}

/* Decoding tables of the 16 contexts: the total M, cumulative frequencies and the symbol of every
 * slot (for the two halves of the joint table, slots relative to each half's start). */
typedef struct {
    const uint16_t* q16;
    uint32_t M;
    int prob_bits;
    uint32_t cum[ORC_NCTX][257];
    uint8_t slot_sym[ORC_NCTX][ORC_M_MAX];
} dtables;

static void build_dtables(const uint16_t* q16, int prob_bits, dtables* T)
{
    T->q16 = q16;
    T->prob_bits = prob_bits;
    T->M = 1u << prob_bits;
    for (int c = 0; c < ORC_NCTX; c++) {
        cumulate(q16 + 256 * c, T->cum[c]);
        memset(T->slot_sym[c], 0, ORC_M_MAX);
        for (int s = 0; s < 256; s++)
            for (uint32_t i = T->cum[c][s]; i < T->cum[c][s + 1] && i < T->M; i++) T->slot_sym[c][i] = (uint8_t)s;
    }
}

/*
 * Decode one tile of nvec vectors with prepared tables.  Writes sym9 / raw8 as orc_encode_tile
 * reads them and the 32 final states.  rANS decode [ANS]: slot = x mod M, s = the symbol with
 * cum[s] <= slot < cum[s+1], x <- q_s * floor(x / M) + slot - cum[s]; if x < 2^16,
 * x <- x * 2^16 + the lane's next word.  Returns 0 when the tile is consistent (every state back
 * at 2^16, the two lanes of every region meeting exactly, only padding after the last region),
 * 1 when it is not, -1 when a lane's words ran outside the tile.
 */
static int decode_tile(const uint8_t* tile, uint64_t nbytes, int64_t nvec, const dtables* T,
                       uint8_t* sym9, int16_t* raw8, uint32_t* final_states)
{
    if (nbytes < ORC_TILE_HEAD) return -1;
    int64_t nwords = (int64_t)(nbytes - ORC_TILE_HEAD) / 2;
    const uint8_t* words = tile + ORC_TILE_HEAD;
    int64_t start[ORC_PAIRS], count[ORC_PAIRS], total = 0;
    for (int p = 0; p < ORC_PAIRS; p++) {
        count[p] = get16(tile + 4 * ORC_LANES + 2 * p);
        start[p] = total;
        total += count[p];
    }
    if (total > nwords) return -1;
    int64_t nsteps = (nvec + ORC_LANES - 1) / ORC_LANES;
    int64_t used[ORC_LANES];
    int bad = 0;
    for (int l = 0; l < ORC_LANES; l++) {
        int p = l / 2, fwd = (l % 2) == 0;
        uint32_t x = get32(tile + 4 * l);
        int64_t n = 0;   /* words this lane has read */
        for (int64_t k = 0; k < nsteps; k++) {
            int64_t v = k * ORC_LANES + l;
            if (v >= nvec) continue;
            for (int j = 1; j <= 8; j++) {
                uint32_t slot = x & (T->M - 1);
                int c, s;
                if (j == 1) {                    /* (coset, f1): coset 1's slots follow coset 0's */
                    uint32_t tot0 = T->cum[0][256];
                    c = slot < tot0 ? 0 : 1;
                    s = T->slot_sym[context_of(1, c)][c ? slot - tot0 : slot];
                    sym9[v * 9] = (uint8_t)c;
                } else {
                    c = sym9[v * 9];
                    s = T->slot_sym[context_of(j, c)][slot];
                }
                uint32_t q, cm;
                freq_cum(T->q16, T->cum, j, c, s, &q, &cm);
                x = q * (x / T->M) + slot - cm;
                sym9[v * 9 + j] = (uint8_t)s;
                if (x < ORC_L) {
                    int64_t w = fwd ? start[p] + n : start[p] + count[p] - 1 - n;
                    if (n >= count[p]) return -1;
                    x = (x << 16) | get16(words + 2 * w);
                    n++;
                }
            }
            for (int j = 1; j <= 8; j++)
                if (sym9[v * 9 + j] == ORC_ESC) {
                    int64_t w = fwd ? start[p] + n : start[p] + count[p] - 1 - n;
                    if (n >= count[p]) return -1;
                    raw8[v * 8 + (j - 1)] = (int16_t)get16(words + 2 * w);
                    n++;
                }
        }
        used[l] = n;
        if (final_states) final_states[l] = x;
        if (x != ORC_L) bad = 1;
    }
    for (int p = 0; p < ORC_PAIRS; p++)
        if (used[2 * p] + used[2 * p + 1] != count[p]) bad = 1;
    if (nbytes - ORC_TILE_HEAD - 2u * (uint64_t)total >= 16u) bad = 1;
    return bad;
}

/* Decode one tile given the 16 x 256 frequency tables (exposed for the rANS checks). */
int orc_decode_tile(const uint8_t* tile, uint64_t nbytes, int64_t nvec, const uint16_t* q16, int prob_bits,
                    uint8_t* sym9, int16_t* raw8, uint32_t* final_states)
{
    dtables* T = (dtables*)malloc(sizeof(dtables));
    if (!T) return -2;
    build_dtables(q16, prob_bits, T);
    int rc = decode_tile(tile, nbytes, nvec, T, sym9, raw8, final_states);
    free(T);
    return rc;
}

/* ------------------------------------------------------------------------------------------ */
/* The encoder: normalise, quantise, choose the scale, fit row scales, code ([DOC-LQ/RS/ER]).  */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    int dtype;
    int64_t rows, cols, cols_p, vpr;   /* vpr = vectors per row = cols_p / 8 */
    double* w;                         /* rows x cols, exact values            */
    double* rms;                       /* per-row root mean square             */
} matrix;

/* reading: columns are padded with zeros to a multiple of 8; the padding is quantised with the
 * row but is excluded from the RMS and least-squares sums and never written back. */
static double elem(const matrix* m, int64_t r, int64_t c) { return c < m->cols ? m->w[r * m->cols + c] : 0.0; }

/* [DOC-LQ]: every row is first divided by its RMS. */
static void row_rms(matrix* m)
{
    for (int64_t r = 0; r < m->rows; r++) {
        double acc = 0.0;
        for (int64_t c = 0; c < m->cols; c++) acc += m->w[r * m->cols + c] * m->w[r * m->cols + c];
        m->rms[r] = sqrt(acc / (double)m->cols);
    }
}

/*
 * Quantise vector k of row r at shared scale s: t = clamp(x_hat / s, +-32764) with x_hat the
 * RMS-normalised row, then the E8 nearest point ([DOC-LQ]: the normalised row is cut into
 * 8-vectors, each snapped to the closest point of E8 dilated by one scale s common to the whole
 * tensor).  An all-zero row (RMS 0) maps every vector to the origin.
 */
static void quantise_vector(const matrix* m, int64_t r, int64_t k, double s, double y[8], int* coset)
{
    double t[8];
    for (int i = 0; i < 8; i++) {
        double xh = m->rms[r] > 0.0 ? elem(m, r, 8 * k + i) / m->rms[r] : 0.0;
        double v = xh / s;
        if (v > ORC_CLAMP) v = ORC_CLAMP;
        if (v < -ORC_CLAMP) v = -ORC_CLAMP;
        t[i] = v;
    }
    orc_e8_nearest(t, y, coset);
}

/* A quantised vector's coset and field symbols (9 values; the coset is coded with f1) and the raw
 * values of escaped fields. */
static void vector_symbols(const double y[8], int coset, uint8_t sym[9], int16_t raw[8])
{
    int32_t f[8];
    orc_point_to_fields(y, coset, f);
    sym[0] = (uint8_t)coset;
    for (int j = 0; j < 8; j++) {
        sym[1 + j] = (uint8_t)field_symbol(f[j]);
        raw[j] = (int16_t)f[j];
    }
}

/* reading: S = clamp(next_pow2(ceil(128 / target)), 16, 1024) steps per tile, unless given. */
static int64_t default_steps(double target)
{
    double want = ceil(128.0 / target);
    int64_t s = 1;
    while ((double)s < want) s *= 2;
    if (s < 16) s = 16;
    if (s > 1024) s = 1024;
    return s;
}

/* Bytes of the serialised table section for the given 16 tables (unpadded). */
static uint64_t table_section_bytes(const uint16_t* q16)
{
    uint64_t bytes = 0;
    for (int ctx = 0; ctx < ORC_NCTX; ctx++) {
        const uint16_t* q = q16 + 256 * ctx;
        int lo = -1, hi = -1;
        for (int s = 0; s < ORC_ESC; s++)
            if (q[s]) { if (lo < 0) lo = s; hi = s; }
        bytes += 4 + (lo < 0 ? 0 : 2u * (uint64_t)(hi - lo + 1));
    }
    return bytes;
}

/* Metadata bytes of a blob with these tables: the exact header, table, row-scale, row-maximum and
 * tile-offset sections, plus per tile its 160 header bytes (states, region counts) and 8 bytes,
 * the mean padding. */
static double metadata_bytes(const uint16_t* q16, int64_t rows, int64_t ntiles)
{
    return (double)(ORC_HEADER + pad16(table_section_bytes(q16)) + pad16(4u * (uint64_t)rows) +
                    pad16(2u * (uint64_t)rows) + pad16(4u * (uint64_t)(ntiles + 1))) +
           (double)ntiles * (160.0 + 8.0);
}

/*
 * Estimated blob size in bits per element at scale s from the sampled rows ([DOC-RS]: a
 * candidate scale is judged by the predicted size of its coded fields plus the metadata the
 * decoder needs).
 * reading: n_s = min(rows, 256) rows at floor(i * rows / n_s); tables are quantised from the
 * sample's counts; coded size = sum over contexts and symbols of n * -log2(q / M) bits plus
 * 16 bits per escape, scaled by rows / n_s; metadata as metadata_bytes counts it.
 * With full_sample != 0 every row is used (n_s = rows).
 */
static double estimate_bpp(const matrix* m, double s, int64_t S, int full_sample, int prob_bits)
{
    int64_t ns = full_sample ? m->rows : (m->rows < 256 ? m->rows : 256);
    uint64_t* cnt = (uint64_t*)calloc(ORC_NCTX * 256, sizeof(uint64_t));
    uint64_t nesc = 0;
    for (int64_t i = 0; i < ns; i++) {
        int64_t r = (int64_t)((i * m->rows) / ns);
        for (int64_t k = 0; k < m->vpr; k++) {
            double y[8];
            int c;
            uint8_t sym[9];
            int16_t raw[8];
            quantise_vector(m, r, k, s, y, &c);
            vector_symbols(y, c, sym, raw);
            for (int u = 1; u <= 8; u++) {
                cnt[256 * context_of(u, c) + sym[u]]++;
                if (u > 0 && sym[u] == ORC_ESC) nesc++;
            }
        }
    }
    uint16_t q16[ORC_NCTX * 256];
    build_tables16(cnt, q16, prob_bits);
    const double M = (double)(1u << prob_bits);
    double bits = 0.0;
    for (int ctx = 0; ctx < ORC_NCTX; ctx++)
        for (int sy = 0; sy < 256; sy++)
            if (cnt[256 * ctx + sy]) bits += (double)cnt[256 * ctx + sy] * -log2((double)q16[256 * ctx + sy] / M);
    double payload = ((double)m->rows / (double)ns) * (bits / 8.0 + 2.0 * (double)nesc);
    int64_t V = m->rows * m->vpr;
    int64_t ntiles = (V + 32 * S - 1) / (32 * S);
    double meta = metadata_bytes(q16, m->rows, ntiles);
    free(cnt);
    return 8.0 * (meta + payload) / ((double)m->rows * (double)m->cols);
}

/*
 * Choose the shared scale ([DOC-RS]: the scale is searched for on a sample of rows;
 * [DOC-LQ]: finer spacing costs more bits).
 * reading: the finest scale whose estimate meets the target, by 48 bisection steps on log2 s
 * over [-24, 8]; if even 2^8 misses the target, 2^8 (the actual size is reported as it is,
 * [DOC-ER]: the stored rate need not equal the requested one).
 */
static double choose_scale(const matrix* m, double target, int64_t S, int prob_bits)
{
    double lo = -24.0, hi = 8.0;
    if (estimate_bpp(m, exp2(hi), S, 0, prob_bits) > target) return exp2(hi);
    if (estimate_bpp(m, exp2(lo), S, 0, prob_bits) <= target) return exp2(lo);
    for (int it = 0; it < 48; it++) {
        double mid = 0.5 * (lo + hi);
        if (estimate_bpp(m, exp2(mid), S, 0, prob_bits) <= target) hi = mid;
        else lo = mid;
    }
    return exp2(hi);
}

static int load_matrix(matrix* m, const void* data, int dtype, int64_t rows, int64_t cols)
{
    if (rows <= 0 || cols <= 0 || dtype_size(dtype) == 0) return -1;
    m->dtype = dtype;
    m->rows = rows;
    m->cols = cols;
    m->cols_p = (cols + 7) / 8 * 8;
    m->vpr = m->cols_p / 8;
    m->w = (double*)malloc((size_t)(rows * cols) * sizeof(double));
    m->rms = (double*)malloc((size_t)rows * sizeof(double));
    if (!m->w || !m->rms) return -2;
    for (int64_t i = 0; i < rows * cols; i++) {
        m->w[i] = orc_dtype_to_f64(load_bits(data, dtype, (uint64_t)i), dtype);
        if (!isfinite(m->w[i])) return -3;
    }
    row_rms(m);
    return 0;
}

static void free_matrix(matrix* m)
{
    free(m->w);
    free(m->rms);
}

/* Estimated bits per element at a given scale (exposed for the size-estimate check). */
double orc_estimate_bpp(const void* data, int dtype, int64_t rows, int64_t cols, double scale,
                        int64_t S, int full_sample, int prob_bits)
{
    if (prob_bits == 0) prob_bits = ORC_PB_DEFAULT;
    if (prob_bits != 10 && prob_bits != 12) return -1.0;
    matrix m;
    memset(&m, 0, sizeof m);
    if (load_matrix(&m, data, dtype, rows, cols)) { free_matrix(&m); return -1.0; }
    double b = estimate_bpp(&m, scale, S, full_sample, prob_bits);
    free_matrix(&m);
    return b;
}

/* ------------------------------------------------------------------------------------------ */
/* Per-row rate-distortion refinement ([DOC-RS]: optional and off by default; several           */
/* resolutions are compared for every row and handed out under the estimated storage budget,    */
/* alternating the choice with updates of the shared probability model).                        */
/*                                                                                            */
/* reading: the candidates of row r are s_r = s * 2^(k/2) for k in {0, -1, 1, -2, 2} (in this   */
/* order, which breaks ties), s the searched shared scale.  For each candidate:                 */
/*   D = sum over real columns of (w - alpha * y)^2, alpha the row's fp32 least-squares scale   */
/*       at that resolution (what the decoder multiplies by), in fp64;                          */
/*   R = sum over the row's symbols of -log2(q / M) under the current tables (log2 M for a      */
/*       symbol they do not hold) plus 16 bits per escape.                                      */
/* A round picks k_r = argmin D + lambda R for every row, with lambda = 2^u the smallest, by 64 */
/* bisection steps on u over [-100, 40], whose total R meets the budget                        */
/* target * rows * cols - 8 * (metadata bytes, counted as the size estimate counts them); 0 if  */
/* even the finest choices meet it.  The tables are then rebuilt from the chosen quantisations. */
/* Three rounds, starting from tables of k = 0 everywhere.  The decode format is unchanged: a   */
/* row's resolution is absorbed by its least-squares scale.                                     */
/* ------------------------------------------------------------------------------------------ */

#define RD_NK 5
#define RD_ROUNDS 3
static const int rd_k[RD_NK] = {0, -1, 1, -2, 2};

static double rd_resolution(double s, int ki) { return s * exp2(0.5 * rd_k[ki]); }

/* Quantise row r at scale sr: its symbols (vpr x 9) and escape count; returns D. */
static double rd_row(const matrix* m, int64_t r, double sr, uint8_t* sym, uint64_t* nesc)
{
    double swy = 0.0, syy = 0.0;
    double* ys = (double*)malloc((size_t)m->vpr * 8 * sizeof(double));
    *nesc = 0;
    for (int64_t k = 0; k < m->vpr; k++) {
        int c;
        int16_t raw[8];
        quantise_vector(m, r, k, sr, ys + 8 * k, &c);
        vector_symbols(ys + 8 * k, c, sym + 9 * k, raw);
        for (int j = 1; j <= 8; j++) *nesc += sym[9 * k + j] == ORC_ESC;
        for (int i = 0; i < 8; i++)
            if (8 * k + i < m->cols) {
                swy += elem(m, r, 8 * k + i) * ys[8 * k + i];
                syy += ys[8 * k + i] * ys[8 * k + i];
            }
    }
    float a = syy > 0.0 ? (float)(swy / syy) : 0.0f;
    double d = 0.0;
    for (int64_t k = 0; k < m->vpr; k++)
        for (int i = 0; i < 8; i++)
            if (8 * k + i < m->cols) {
                double e = elem(m, r, 8 * k + i) - (double)a * ys[8 * k + i];
                d += e * e;
            }
    free(ys);
    return d;
}

/* Symbol counts of the rows at their chosen candidates. */
static void rd_counts(const matrix* m, const uint8_t* sym, const int* kr, uint64_t* cnt)
{
    memset(cnt, 0, ORC_NCTX * 256 * sizeof(uint64_t));
    for (int64_t r = 0; r < m->rows; r++) {
        const uint8_t* sr = sym + ((size_t)r * RD_NK + (size_t)kr[r]) * (size_t)m->vpr * 9;
        for (int64_t k = 0; k < m->vpr; k++)
            for (int u = 1; u <= 8; u++) cnt[256 * context_of(u, sr[9 * k]) + sr[9 * k + u]]++;
    }
}

/* Row choices k_r (indexes into rd_k) for the given lambda; returns the total rate. */
static double rd_choose(const matrix* m, const double* D, const double* R, double lambda, int* kr)
{
    double total = 0.0;
    for (int64_t r = 0; r < m->rows; r++) {
        int best = 0;
        double bc = D[r * RD_NK] + lambda * R[r * RD_NK];
        for (int ki = 1; ki < RD_NK; ki++) {
            double c = D[r * RD_NK + ki] + lambda * R[r * RD_NK + ki];
            if (c < bc) { bc = c; best = ki; }
        }
        kr[r] = best;
        total += R[r * RD_NK + best];
    }
    return total;
}

/* The refinement: fills kr[rows] with each row's candidate index.  Returns 0 or -2 (memory). */
static int rd_allocate(const matrix* m, double s, double target, int64_t S, int prob_bits, int* kr)
{
    const double M = (double)(1u << prob_bits);
    const size_t per = (size_t)m->vpr * 9;
    uint8_t* sym = (uint8_t*)malloc((size_t)m->rows * RD_NK * per);
    uint64_t* nesc = (uint64_t*)malloc((size_t)m->rows * RD_NK * sizeof(uint64_t));
    double* D = (double*)malloc((size_t)m->rows * RD_NK * sizeof(double));
    double* R = (double*)malloc((size_t)m->rows * RD_NK * sizeof(double));
    uint64_t* cnt = (uint64_t*)malloc(ORC_NCTX * 256 * sizeof(uint64_t));
    int rc = 0;
    if (!sym || !nesc || !D || !R || !cnt) { rc = -2; goto out; }
    for (int64_t r = 0; r < m->rows; r++)
        for (int ki = 0; ki < RD_NK; ki++)
            D[r * RD_NK + ki] = rd_row(m, r, rd_resolution(s, ki), sym + ((size_t)r * RD_NK + ki) * per,
                                       &nesc[r * RD_NK + ki]);
    for (int64_t r = 0; r < m->rows; r++) kr[r] = 0;
    {
        int64_t V = m->rows * m->vpr;
        int64_t ntiles = (V + 32 * S - 1) / (32 * S);
        for (int round = 0; round < RD_ROUNDS; round++) {
            uint16_t q16[ORC_NCTX * 256];
            double cost[ORC_NCTX * 256];
            rd_counts(m, sym, kr, cnt);
            build_tables16(cnt, q16, prob_bits);
            for (int i = 0; i < ORC_NCTX * 256; i++)
                cost[i] = q16[i] ? -log2((double)q16[i] / M) : log2(M);
            for (int64_t r = 0; r < m->rows; r++)
                for (int ki = 0; ki < RD_NK; ki++) {
                    const uint8_t* sr = sym + ((size_t)r * RD_NK + ki) * per;
                    double bits = 16.0 * (double)nesc[r * RD_NK + ki];
                    for (int64_t k = 0; k < m->vpr; k++)
                        for (int u = 1; u <= 8; u++) bits += cost[256 * context_of(u, sr[9 * k]) + sr[9 * k + u]];
                    R[r * RD_NK + ki] = bits;
                }
            double meta = metadata_bytes(q16, m->rows, ntiles);
            double budget = target * (double)m->rows * (double)m->cols - 8.0 * meta;
            if (rd_choose(m, D, R, 0.0, kr) > budget) {
                double lo = -100.0, hi = 40.0;
                if (rd_choose(m, D, R, exp2(hi), kr) <= budget) {
                    for (int it = 0; it < 64; it++) {
                        double mid = 0.5 * (lo + hi);
                        if (rd_choose(m, D, R, exp2(mid), kr) <= budget) hi = mid;
                        else lo = mid;
                    }
                }
                rd_choose(m, D, R, exp2(hi), kr);
            }
        }
    }
out:
    free(sym);
    free(nesc);
    free(D);
    free(R);
    free(cnt);
    return rc;
}

/*
 * Compress a rows x cols matrix stored as dtype bits.  steps_per_tile = 0 selects the default S;
 * scale_override > 0 skips the search; prob_bits is 12 or 10 (0 selects 12).  On success *blob is
 * a malloc'd byte string of *len bytes.
 *
 * Blob layout (little-endian, every section 16-byte aligned; [DOC-ER]: besides the coded fields
 * the blob keeps the frequency tables, the per-row scales and per-tile bookkeeping):
 *   header (96 bytes): "EPK1", u16 version 4, u8 dtype, u8 R, u64 rows, u64 cols, u32 S,
 *     u32 n_tiles, f64 s, u64 total bytes, u64 offsets of the table, row-scale, tile-offset
 *     and stream sections, u64 offset of the row-maximum section, u8 prob_bits, 7 zero bytes;
 *   tables: for c = 0,1 and j = 1..8: u16 q(escape), u8 lo, u8 n, u16 q[lo .. lo+n-1]
 *     (symbols 0..254); the two j = 1 tables are the coset halves of the joint (c, f1) table;
 *   row scales: f32 per row;
 *   row maxima: u16 per row, the largest |2 y| over the row's real columns (2 y is an integer:
 *     the lattice coordinates are integers or half-integers, |y| <= 32764.5);
 *   tile offsets: u32[n_tiles + 1], in 16-byte units from the stream section start;
 *   stream: the tiles.
 */
int orc_compress_ex(const void* data, int dtype, int64_t rows, int64_t cols, double target_bpp,
                    int64_t steps_per_tile, double scale_override, int rd_refine, int prob_bits, uint8_t** blob,
                    uint64_t* len)
{
    *blob = NULL;
    *len = 0;
    /* [DOC-0]: the target must be finite and within 0.001 to 11 bits per element */
    if (!(target_bpp >= 0.001 && target_bpp <= 11.0)) return -4;
    if (prob_bits == 0) prob_bits = ORC_PB_DEFAULT;
    if (prob_bits != 10 && prob_bits != 12) return -4;
    matrix m;
    memset(&m, 0, sizeof m);
    int rc = load_matrix(&m, data, dtype, rows, cols);
    if (rc) { free_matrix(&m); return rc; }
    if (steps_per_tile > 1024) { free_matrix(&m); return -4; }   /* region counts are u16 */
    int64_t S = steps_per_tile > 0 ? steps_per_tile : default_steps(target_bpp);
    double s = scale_override > 0 ? scale_override : choose_scale(&m, target_bpp, S, prob_bits);
    int* kr = NULL;                      /* per-row candidate of the refinement, when enabled */
    if (rd_refine) {
        kr = (int*)malloc((size_t)rows * sizeof(int));
        if (!kr || rd_allocate(&m, s, target_bpp, S, prob_bits, kr)) { free(kr); free_matrix(&m); return -2; }
    }

    /* Quantise the whole tensor at s; fit one least-squares scale per row ([DOC-RS]: with s
     * fixed, every row is quantised and gets its own reconstruction scale by least squares):
     * alpha_r = sum w y / sum y^2 over real columns, stored as fp32 (0 when sum y^2 = 0); and
     * keep each row's largest |2 y| over its real columns. */
    int64_t V = rows * m.vpr;
    uint8_t* sym9 = (uint8_t*)malloc((size_t)V * 9);
    int16_t* raw8 = (int16_t*)malloc((size_t)V * 8 * sizeof(int16_t));
    float* alpha = (float*)malloc((size_t)rows * sizeof(float));
    uint32_t* rowmax = (uint32_t*)calloc((size_t)rows, sizeof(uint32_t));
    uint64_t* cnt = (uint64_t*)calloc(ORC_NCTX * 256, sizeof(uint64_t));
    for (int64_t r = 0; r < rows; r++) {
        double swy = 0.0, syy = 0.0;
        for (int64_t k = 0; k < m.vpr; k++) {
            double y[8];
            int c;
            int64_t v = r * m.vpr + k;
            quantise_vector(&m, r, k, kr ? rd_resolution(s, kr[r]) : s, y, &c);
            vector_symbols(y, c, sym9 + 9 * v, raw8 + 8 * v);
            for (int i = 0; i < 8; i++)
                if (8 * k + i < cols) {
                    swy += elem(&m, r, 8 * k + i) * y[i];
                    syy += y[i] * y[i];
                    uint32_t a2 = (uint32_t)fabs(2.0 * y[i]);
                    if (a2 > rowmax[r]) rowmax[r] = a2;
                }
            for (int u = 1; u <= 8; u++) cnt[256 * context_of(u, c) + sym9[9 * v + u]]++;
        }
        alpha[r] = syy > 0.0 ? (float)(swy / syy) : 0.0f;
    }

    /* Probability tables from the whole tensor ([DOC-LQ]: one model per coordinate field, given
     * the coset). */
    uint16_t q16[ORC_NCTX * 256];
    build_tables16(cnt, q16, prob_bits);

    /* Tiles. */
    int64_t per_tile = 32 * S;
    int64_t ntiles = (V + per_tile - 1) / per_tile;
    uint64_t* tsize = (uint64_t*)malloc((size_t)(ntiles + 1) * sizeof(uint64_t));
    uint64_t stream_bytes = 0;
    for (int64_t t = 0; t < ntiles; t++) {
        int64_t v0 = t * per_tile, nv = V - v0 < per_tile ? V - v0 : per_tile;
        tsize[t] = orc_encode_tile(sym9 + 9 * v0, raw8 + 8 * v0, nv, q16, prob_bits, NULL, 0);
        if (tsize[t] == 0) { rc = -5; goto done; }
        stream_bytes += tsize[t];
    }

    /* Serialise. */
    {
        uint64_t tab_bytes = table_section_bytes(q16);
        uint64_t off_tab = ORC_HEADER;
        uint64_t off_alpha = off_tab + pad16(tab_bytes);
        uint64_t off_rmax = off_alpha + pad16(4u * (uint64_t)rows);
        uint64_t off_offs = off_rmax + pad16(2u * (uint64_t)rows);
        uint64_t off_stream = off_offs + pad16(4u * (uint64_t)(ntiles + 1));
        uint64_t total = off_stream + stream_bytes;
        uint8_t* b = (uint8_t*)calloc((size_t)total, 1);
        if (!b) { rc = -2; goto done; }
        memcpy(b, "EPK1", 4);
        put16(b + 4, ORC_VERSION);
        b[6] = (uint8_t)dtype;
        b[7] = ORC_R;
        put64(b + 8, (uint64_t)rows);
        put64(b + 16, (uint64_t)cols);
        put32(b + 24, (uint32_t)S);
        put32(b + 28, (uint32_t)ntiles);
        memcpy(b + 32, &s, 8);                                     /* f64, little-endian host */
        put64(b + 40, total);
        put64(b + 48, off_tab);
        put64(b + 56, off_alpha);
        put64(b + 64, off_offs);
        put64(b + 72, off_stream);
        put64(b + 80, off_rmax);
        b[88] = (uint8_t)prob_bits;
        uint8_t* p = b + off_tab;
        for (int ctx = 0; ctx < ORC_NCTX; ctx++) {
            const uint16_t* q = q16 + 256 * ctx;
            int lo = -1, hi = -1;
            for (int sy = 0; sy < ORC_ESC; sy++)
                if (q[sy]) { if (lo < 0) lo = sy; hi = sy; }
            int n = lo < 0 ? 0 : hi - lo + 1;
            put16(p, q[ORC_ESC]);
            p[2] = (uint8_t)(lo < 0 ? 0 : lo);
            p[3] = (uint8_t)n;
            p += 4;
            for (int i = 0; i < n; i++, p += 2) put16(p, q[lo + i]);
        }
        for (int64_t r = 0; r < rows; r++) {
            uint32_t ab;
            memcpy(&ab, &alpha[r], 4);
            put32(b + off_alpha + 4 * r, ab);
            put16(b + off_rmax + 2 * r, rowmax[r]);
        }
        uint64_t acc = 0;
        for (int64_t t = 0; t <= ntiles; t++) {
            put32(b + off_offs + 4 * t, (uint32_t)(acc / 16u));
            if (t < ntiles) acc += tsize[t];
        }
        acc = 0;
        for (int64_t t = 0; t < ntiles; t++) {
            int64_t v0 = t * per_tile, nv = V - v0 < per_tile ? V - v0 : per_tile;
            orc_encode_tile(sym9 + 9 * v0, raw8 + 8 * v0, nv, q16, prob_bits, b + off_stream + acc, tsize[t]);
            acc += tsize[t];
        }
        *blob = b;
        *len = total;
    }
done:
    free(kr);
    free(tsize);
    free(sym9);
    free(raw8);
    free(alpha);
    free(rowmax);
    free(cnt);
    free_matrix(&m);
    return rc;
}

/* orc_compress_ex with the refinement off (the default) and 12-bit totals. */
int orc_compress(const void* data, int dtype, int64_t rows, int64_t cols, double target_bpp,
                 int64_t steps_per_tile, double scale_override, uint8_t** blob, uint64_t* len)
{
    return orc_compress_ex(data, dtype, rows, cols, target_bpp, steps_per_tile, scale_override, 0, 0, blob, len);
}

/* ------------------------------------------------------------------------------------------ */
/* The decoder ([DOC-ER]: fields back to lattice points, times the row scales, in a tensor of  */
/* the original shape and element type).                                                      */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    int dtype, prob_bits;
    int64_t rows, cols, vpr, S, ntiles, V;
    double s;
    uint16_t q16[ORC_NCTX * 256];
    const uint8_t* alpha;
    const uint8_t* rowmax;
    const uint8_t* offs;
    const uint8_t* stream;
    uint64_t off_offs, off_stream, stream_bytes;
} parsed;

static int parse_blob(const uint8_t* b, uint64_t len, parsed* P)
{
    if (len < ORC_HEADER || memcmp(b, "EPK1", 4) != 0 || get16(b + 4) != ORC_VERSION || b[7] != ORC_R) return -6;
    P->dtype = b[6];
    P->prob_bits = b[88];
    if (P->prob_bits != 10 && P->prob_bits != 12) return -6;
    const uint32_t M = 1u << P->prob_bits;
    P->rows = (int64_t)get64(b + 8);
    P->cols = (int64_t)get64(b + 16);
    P->S = get32(b + 24);
    P->ntiles = get32(b + 28);
    memcpy(&P->s, b + 32, 8);
    uint64_t total = get64(b + 40), off_tab = get64(b + 48), off_alpha = get64(b + 56);
    uint64_t off_offs = get64(b + 64), off_stream = get64(b + 72), off_rmax = get64(b + 80);
    if (total != len || P->rows <= 0 || P->cols <= 0 || P->S <= 0 || dtype_size(P->dtype) == 0) return -6;
    P->vpr = (P->cols + 7) / 8;
    P->V = P->rows * P->vpr;
    if (P->ntiles != (P->V + 32 * P->S - 1) / (32 * P->S)) return -6;
    if (off_tab < ORC_HEADER || off_tab > off_alpha || off_alpha + 4u * (uint64_t)P->rows > off_rmax ||
        off_rmax + 2u * (uint64_t)P->rows > off_offs || off_offs + 4u * (uint64_t)(P->ntiles + 1) > off_stream ||
        off_stream > len)
        return -6;
    memset(P->q16, 0, sizeof P->q16);
    const uint8_t* p = b + off_tab;
    for (int ctx = 0; ctx < ORC_NCTX; ctx++) {
        if ((uint64_t)(p + 4 - b) > off_alpha) return -6;
        uint16_t* q = P->q16 + 256 * ctx;
        q[ORC_ESC] = (uint16_t)get16(p);
        int lo = p[2], n = p[3];
        p += 4;
        if (lo + n > ORC_ESC || (uint64_t)(p + 2 * n - b) > off_alpha) return -6;
        for (int i = 0; i < n; i++, p += 2) q[lo + i] = (uint16_t)get16(p);
    }
    uint32_t sums[ORC_NCTX];
    for (int ctx = 0; ctx < ORC_NCTX; ctx++) {
        sums[ctx] = 0;
        for (int sy = 0; sy < 256; sy++) sums[ctx] += P->q16[256 * ctx + sy];
    }
    if (sums[0] + sums[8] != M) return -6;                     /* the joint (coset, f1) table */
    for (int ctx = 0; ctx < ORC_NCTX; ctx++)
        if (ctx != 0 && ctx != 8 && sums[ctx] != 0 && sums[ctx] != M) return -6;
    P->alpha = b + off_alpha;
    P->rowmax = b + off_rmax;
    P->offs = b + off_offs;
    P->stream = b + off_stream;
    P->off_offs = off_offs;
    P->off_stream = off_stream;
    P->stream_bytes = len - off_stream;
    if (get32(P->offs) != 0 || 16u * (uint64_t)get32(P->offs + 4 * P->ntiles) != P->stream_bytes) return -6;
    return 0;
}

/* Decode tiles [t0, t1) to symbols.  sym9 / raw8 hold the vectors of those tiles only (vector
 * t0 * 32S is element 0).  Returns 0, or a negative code for an inconsistent tile. */
static int decode_tiles_to_symbols(const parsed* P, int64_t t0, int64_t t1, uint8_t* sym9, int16_t* raw8)
{
    int64_t per_tile = 32 * P->S, base = t0 * per_tile;
    dtables* T = (dtables*)malloc(sizeof(dtables));
    if (!T) return -2;
    build_dtables(P->q16, P->prob_bits, T);
    int out = 0;
    for (int64_t t = t0; t < t1; t++) {
        uint64_t a = 16u * (uint64_t)get32(P->offs + 4 * t), e = 16u * (uint64_t)get32(P->offs + 4 * (t + 1));
        if (e < a || e > P->stream_bytes) { out = -6; break; }
        int64_t v0 = t * per_tile, nv = P->V - v0 < per_tile ? P->V - v0 : per_tile;
        int rc = decode_tile(P->stream + a, e - a, nv, T, sym9 + 9 * (v0 - base), raw8 + 8 * (v0 - base), NULL);
        if (rc) { out = rc < 0 ? -7 : -8; break; }
    }
    free(T);
    return out;
}

/* Field values of the vectors of tiles [t0, t1): fields[v*9] = coset, fields[v*9 + j] = f_j.
 * The array is indexed by global vector number and has room for all V vectors. */
int orc_decode_fields(const uint8_t* blob, uint64_t len, int64_t t0, int64_t t1, int16_t* fields)
{
    parsed P;
    int rc = parse_blob(blob, len, &P);
    if (rc) return rc;
    if (t1 < 0 || t1 > P.ntiles) t1 = P.ntiles;
    if (t0 < 0 || t0 > t1) return -1;
    int64_t v0 = t0 * 32 * P.S, v1 = t1 * 32 * P.S < P.V ? t1 * 32 * P.S : P.V;
    uint8_t* sym9 = (uint8_t*)calloc((size_t)(v1 - v0) * 9 + 9, 1);
    int16_t* raw8 = (int16_t*)calloc((size_t)(v1 - v0) * 8 + 8, sizeof(int16_t));
    rc = decode_tiles_to_symbols(&P, t0, t1, sym9, raw8);
    if (rc == 0) {
        for (int64_t v = v0; v < v1; v++) {
            const uint8_t* sy9 = sym9 + 9 * (v - v0);
            fields[9 * v] = sy9[0];
            for (int j = 1; j <= 8; j++) {
                int sy = sy9[j];
                fields[9 * v + j] = (int16_t)(sy == ORC_ESC ? raw8[8 * (v - v0) + j - 1] : sy - ORC_R);
            }
        }
    }
    free(sym9);
    free(raw8);
    return rc;
}

/*
 * Decode tiles [t0, t1) (all tiles when t1 < 0) into out, a contiguous rows x cols array of
 * dtype_out; elements of other tiles are left untouched.  Each element is the fp32 product of
 * the row's fp32 scale and the lattice coordinate (exact in fp32), rounded to nearest-even, then
 * rounded to the container (RNE; E4M3 saturates to +-448).
 */
int orc_decompress_tiles(const uint8_t* blob, uint64_t len, int64_t t0, int64_t t1, int dtype_out, void* out)
{
    parsed P;
    int rc = parse_blob(blob, len, &P);
    if (rc) return rc;
    if (dtype_size(dtype_out) == 0) return -1;
    if (t1 < 0 || t1 > P.ntiles) t1 = P.ntiles;
    if (t0 < 0 || t0 > t1) return -1;
    int64_t v0 = t0 * 32 * P.S, v1 = t1 * 32 * P.S < P.V ? t1 * 32 * P.S : P.V;
    uint8_t* sym9 = (uint8_t*)calloc((size_t)(v1 - v0) * 9 + 9, 1);
    int16_t* raw8 = (int16_t*)calloc((size_t)(v1 - v0) * 8 + 8, sizeof(int16_t));
    rc = decode_tiles_to_symbols(&P, t0, t1, sym9, raw8);
    if (rc == 0) {
        for (int64_t v = v0; v < v1; v++) {
            int64_t r = v / P.vpr, k = v % P.vpr;
            int32_t f[8];
            double y[8];
            const uint8_t* sy9 = sym9 + 9 * (v - v0);
            int c = sy9[0];
            for (int j = 1; j <= 8; j++) {
                int sy = sy9[j];
                f[j - 1] = sy == ORC_ESC ? raw8[8 * (v - v0) + j - 1] : sy - ORC_R;
            }
            orc_fields_to_point(c, f, y);
            float a;
            uint32_t ab = get32(P.alpha + 4 * r);
            memcpy(&a, &ab, 4);
            for (int i = 0; i < 8; i++) {
                int64_t col = 8 * k + i;
                if (col >= P.cols) continue;
                store_value(out, (uint64_t)(r * P.cols + col), dtype_out, (double)a * y[i]);
            }
        }
    }
    free(sym9);
    free(raw8);
    return rc;
}

/* Decode the whole blob into a contiguous rows x cols array of dtype_out. */
int orc_decompress(const uint8_t* blob, uint64_t len, int dtype_out, void* out)
{
    return orc_decompress_tiles(blob, len, 0, -1, dtype_out, out);
}

/*
 * FP8 container with a per-row scale ([ABS]: FP8 is one of the containers, and the storage rate
 * is set apart from the numerical precision of the restored weights).
 * reading: the E4M3 payload of row r holds the row normalised to the format's range and sigma_r
 * carries the scale, sigma_r * payload ~ alpha_r * y:
 *   m_r     = the row's largest |2 y| (the blob's row-maximum section),
 *   g_r     = RNE_fp32(896 / m_r), negated when alpha_r < 0; 0 when m_r = 0 or alpha_r = 0,
 *   payload = E4M3(RNE_fp32(y * g_r)), round to nearest even, saturating (|y * g_r| <= 448),
 *   sigma_r = RNE_fp32(|alpha_r| * m_r / 896), i.e. rowmax |alpha_r * y| / 448.
 * Both quotients are rounded once from their exact values (a double quotient of these sizes is
 * never a float rounding tie unless the exact value is one, so rounding it again to float is
 * exact rounding).
 */
static float f32_of(uint32_t bits)
{
    float f;
    memcpy(&f, &bits, 4);
    return f;
}

float orc_row_gain(float alpha, uint32_t m2)
{
    if (m2 == 0 || alpha == 0.0f) return 0.0f;
    float g = f32_of(orc_round_f32(896.0 / (double)m2));
    return alpha < 0.0f ? -g : g;
}

float orc_row_sigma(float alpha, uint32_t m2)
{
    return f32_of(orc_round_f32(fabs((double)alpha) * (double)m2 / 896.0));
}

/* Decode tiles [t0, t1) (all when t1 < 0) into the E4M3 payload (rows x cols, contiguous; other
 * tiles' elements untouched) and write every row's sigma (rows floats). */
int orc_decompress_rowscaled_tiles(const uint8_t* blob, uint64_t len, int64_t t0, int64_t t1, uint8_t* out,
                                   float* sigma)
{
    parsed P;
    int rc = parse_blob(blob, len, &P);
    if (rc) return rc;
    if (t1 < 0 || t1 > P.ntiles) t1 = P.ntiles;
    if (t0 < 0 || t0 > t1) return -1;
    for (int64_t r = 0; r < P.rows; r++)
        sigma[r] = orc_row_sigma(f32_of(get32(P.alpha + 4 * r)), get16(P.rowmax + 2 * r));
    int64_t v0 = t0 * 32 * P.S, v1 = t1 * 32 * P.S < P.V ? t1 * 32 * P.S : P.V;
    uint8_t* sym9 = (uint8_t*)calloc((size_t)(v1 - v0) * 9 + 9, 1);
    int16_t* raw8 = (int16_t*)calloc((size_t)(v1 - v0) * 8 + 8, sizeof(int16_t));
    rc = decode_tiles_to_symbols(&P, t0, t1, sym9, raw8);
    if (rc == 0) {
        for (int64_t v = v0; v < v1; v++) {
            int64_t r = v / P.vpr, k = v % P.vpr;
            int32_t f[8];
            double y[8];
            const uint8_t* sy9 = sym9 + 9 * (v - v0);
            for (int j = 1; j <= 8; j++) {
                int sy = sy9[j];
                f[j - 1] = sy == ORC_ESC ? raw8[8 * (v - v0) + j - 1] : sy - ORC_R;
            }
            orc_fields_to_point(sy9[0], f, y);
            float g = orc_row_gain(f32_of(get32(P.alpha + 4 * r)), get16(P.rowmax + 2 * r));
            for (int i = 0; i < 8; i++) {
                int64_t col = 8 * k + i;
                if (col >= P.cols) continue;
                out[r * P.cols + col] = (uint8_t)orc_f32_to_e4m3(orc_round_f32((double)g * y[i]));
            }
        }
    }
    free(sym9);
    free(raw8);
    return rc;
}

/* [DOC-ER]: the reported rate is 8 x every stored byte (metadata included) / element count. */
double orc_actual_bpp(const uint8_t* blob, uint64_t len)
{
    parsed P;
    if (parse_blob(blob, len, &P)) return -1.0;
    return 8.0 * (double)len / ((double)P.rows * (double)P.cols);
}

/* Header fields, for tests: rows, cols, S, n_tiles, dtype, prob_bits, the byte offsets of the
 * tile-offset and stream sections, and the shared scale. */
int orc_blob_info(const uint8_t* blob, uint64_t len, int64_t* info8, double* scale)
{
    parsed P;
    int rc = parse_blob(blob, len, &P);
    if (rc) return rc;
    info8[0] = P.rows;
    info8[1] = P.cols;
    info8[2] = P.S;
    info8[3] = P.ntiles;
    info8[4] = P.dtype;
    info8[5] = P.prob_bits;
    info8[6] = (int64_t)P.off_offs;
    info8[7] = (int64_t)P.off_stream;
    *scale = P.s;
    return 0;
}

void orc_free(void* p) { free(p); }

/* ------------------------------------------------------------------------------------------ */
/* Array forms of the per-vector functions, for the checks (one call per array).              */
/* ------------------------------------------------------------------------------------------ */

void orc_e8_nearest_n(const double* t, int64_t n, double* y, int32_t* coset)
{
    for (int64_t i = 0; i < n; i++) {
        int c;
        orc_e8_nearest(t + 8 * i, y + 8 * i, &c);
        coset[i] = c;
    }
}

void orc_point_to_fields_n(const double* y, const int32_t* coset, int64_t n, int32_t* f)
{
    for (int64_t i = 0; i < n; i++) orc_point_to_fields(y + 8 * i, coset[i], f + 8 * i);
}

void orc_fields_to_point_n(const int32_t* coset, const int32_t* f, int64_t n, double* y)
{
    for (int64_t i = 0; i < n; i++) orc_fields_to_point(coset[i], f + 8 * i, y + 8 * i);
}

void orc_dtype_to_f64_n(const void* data, int dtype, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_dtype_to_f64(load_bits(data, dtype, (uint64_t)i), dtype);
}

/* fp32 rounding of exact products a[i] * b[i] (double), returned as fp32 bit patterns. */
void orc_round_f32_n(const double* v, int64_t n, uint32_t* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = orc_round_f32(v[i]);
}
