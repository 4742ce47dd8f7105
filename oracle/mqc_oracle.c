/*
 * mqc_oracle.c -- plain, slow, obviously-correct CPU reference for the
 * MicroQonv hot path ("MicroQonv: Reshaping Convolution Tensors for Efficient
 * Microscaling in Training and Inference", arXiv:2609.28358).
 *
 * THIS FILE IS TEST INFRASTRUCTURE.  Only the tests, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header,
 * table or constant with the CUDA library, and the CUDA library never calls it.
 *
 * Everything here is computed in double precision (or exact integer work) in
 * the plainest loop order that follows the definitions:
 *
 *   - MX element formats E4M3 / E5M2 / E2M1: decode tables enumerated from the
 *     bit fields (the maxima 448 and 6 are named in the paper, section III-A,
 *     text of Eq. 4; the field layouts are those of the OCP MX v1.0 / OCP FP8
 *     specifications).
 *   - Shared E8M0 block scale: the power of two of the original microscaling
 *     format (paper, section II-D), with exponent floor(log2(amax)) - emax_elem
 *     (OCP MX rule), clamped to [-127, 127]; amax == 0 gives code 0x00.
 *   - Element encoding: the finite code nearest to x * 2^-e, ties to the code
 *     with an even mantissa LSB (round-to-nearest-even), values beyond the
 *     largest finite magnitude saturate to it; the sign of zero is kept.
 *   - Quantization directions (paper, section IV-B): blocks of 32 along the
 *     A-axis (C_in for X and W, C_out for G_Y), along the B-axis (N for X and
 *     G_Y, C_out for W), or a 32x32 square over (B, A) sharing one scale.
 *   - Channel-batch-first layout (paper, section IV-A, Fig. 3): every spatial
 *     position (h, w) holds a contiguous (B x A) block of codes.
 *   - Naive im2col (paper, section II-C1) and channel-batch-first im2col on
 *     codes and scales (section IV-A).
 *   - Direct convolution forward (Eq. 1), input gradient (Eq. 2) and weight
 *     gradient (Eq. 3), as cross-correlation with stride and zero padding,
 *     each also returning sum |a*b| of its dot product.
 *   - Stochastic rounding of the elements (section III-A, Eq. 6: the
 *     gradients are rounded stochastically), with random bits from the
 *     Philox4x64-10 counter-based generator (Salmon et al., SC 2011).
 *   - NVFP4 (section III-A, Eq. 4-6): per-tensor FP32 scale, E4M3 scale per
 *     block of 16, E2M1 elements, evaluated step by step in fp32.
 *   - The per-element quantization-count and stored-bytes model behind
 *     Table I (section IV-C).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_E4M3 = 0, OR_E5M2 = 1, OR_E2M1 = 2 };
enum { OR_A32 = 0, OR_B32 = 1, OR_SQ32 = 2 };
enum { OR_ORDER_BA = 0, OR_ORDER_AB = 1 };

/* ------------------------------------------------------------------------ */
/* Element formats                                                           */
/* ------------------------------------------------------------------------ */

static int fmt_bits(int fmt) { return fmt == OR_E2M1 ? 4 : 8; }
static int fmt_ebits(int fmt) { return fmt == OR_E4M3 ? 4 : (fmt == OR_E5M2 ? 5 : 2); }
static int fmt_mbits(int fmt) { return fmt == OR_E4M3 ? 3 : (fmt == OR_E5M2 ? 2 : 1); }
static int fmt_bias(int fmt) { return fmt == OR_E4M3 ? 7 : (fmt == OR_E5M2 ? 15 : 1); }

/* Largest normal exponent of the element format (OCP MX "emax_elem"). */
int oracle_emax_elem(int fmt) { return fmt == OR_E4M3 ? 8 : (fmt == OR_E5M2 ? 15 : 2); }

int oracle_fmt_bits(int fmt) { return fmt_bits(fmt); }

/* Value of one element code, from its sign / exponent / mantissa fields.
 * *finite is set to 0 for the Inf and NaN encodings (E4M3 has only the NaN
 * pattern S.1111.111; E5M2 reserves exponent field 31; E2M1 has none). */
double oracle_decode(int fmt, int code, int *finite)
{
    int nb = fmt_bits(fmt), eb = fmt_ebits(fmt), mb = fmt_mbits(fmt), bias = fmt_bias(fmt);
    int sign = (code >> (nb - 1)) & 1;
    int ef = (code >> mb) & ((1 << eb) - 1);
    int m = code & ((1 << mb) - 1);
    *finite = 1;
    if (fmt == OR_E4M3 && ef == 15 && m == 7) { *finite = 0; return NAN; }
    if (fmt == OR_E5M2 && ef == 31) { *finite = 0; return m ? NAN : (sign ? -INFINITY : INFINITY); }
    double mag;
    if (ef == 0) mag = ldexp((double)m, 1 - bias - mb);                 /* subnormal */
    else         mag = ldexp((double)((1 << mb) + m), ef - bias - mb);  /* normal */
    return sign ? -mag : mag;
}

/* Non-negative finite codes in increasing magnitude.  In these sign-magnitude
 * formats the magnitude grows with the code, so the table is just the codes
 * 0, 1, 2, ... up to the last finite one. */
typedef struct { int n; int code[128]; double val[128]; } or_table;

static void build_table(int fmt, or_table *t)
{
    int nb = fmt_bits(fmt);
    t->n = 0;
    for (int c = 0; c < (1 << (nb - 1)); ++c) {
        int fin;
        double v = oracle_decode(fmt, c, &fin);
        if (!fin) continue;
        t->code[t->n] = c;
        t->val[t->n] = v;
        t->n++;
    }
}

static or_table g_tab[3];

/* Filled once when the library is loaded, before any (threaded) use. */
__attribute__((constructor)) static void init_tables(void)
{
    for (int f = 0; f < 3; ++f) build_table(f, &g_tab[f]);
}

static const or_table *table_of(int fmt) { return &g_tab[fmt]; }

/* Largest finite magnitude of the element format (448, 57344, 6). */
double oracle_max_finite(int fmt)
{
    const or_table *t = table_of(fmt);
    return t->val[t->n - 1];
}

/* Encode a real value: the finite code nearest to v, ties to the even code
 * (round-to-nearest-even), saturating beyond the largest finite magnitude,
 * sign of zero kept.  The nearest code is found by bracketing |v| between two
 * neighbouring table entries (binary search over the monotone table). */
int oracle_encode(int fmt, double v)
{
    const or_table *t = table_of(fmt);
    int nb = fmt_bits(fmt);
    if (v != v) return fmt == OR_E2M1 ? 0x7 : 0x7F; /* NaN: never compared */
    int sign = signbit(v) ? 1 : 0;
    double a = fabs(v);
    int code;
    if (a >= t->val[t->n - 1]) {
        code = t->code[t->n - 1];                     /* saturate */
    } else {
        int lo = 0, hi = t->n - 1;                    /* val[lo] <= a < val[hi] */
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (t->val[mid] <= a) lo = mid; else hi = mid;
        }
        double dlo = a - t->val[lo], dhi = t->val[hi] - a;
        if (dlo < dhi) code = t->code[lo];
        else if (dhi < dlo) code = t->code[hi];
        else code = (t->code[lo] & 1) ? t->code[hi] : t->code[lo];  /* tie: even */
    }
    return (sign << (nb - 1)) | code;
}

/* Shared E8M0 scale code of a block with absolute maximum amax:
 * e = floor(log2(amax)) - emax_elem, clamped to [-127, 127], code = e + 127.
 * amax == 0 -> 0x00 (2^-127); a non-finite amax -> 0xFF (the E8M0 NaN). */
int oracle_scale_code(int fmt, double amax)
{
    if (amax != amax || isinf(amax)) return 0xFF;
    if (amax == 0.0) return 0x00;
    int ex;
    frexp(amax, &ex);              /* amax = f * 2^ex with f in [0.5, 1) */
    int e = (ex - 1) - oracle_emax_elem(fmt);
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e + 127;
}

/* ------------------------------------------------------------------------ */
/* Channel-batch-first quantized layout                                      */
/* ------------------------------------------------------------------------ */
/*
 * A source tensor is 4-D [d0][d1][d2][d3] (NCHW-like) with element strides.
 * d0 is the B-axis (N for X and G_Y, C_out for W), d1 the A-axis (C_in for X
 * and W, C_out for G_Y), (d2, d3) the spatial position.
 *
 * Codes are stored per spatial position as a (B x A) block:
 *   order BA (A innermost): codes[((h*d3 + w)*Bp + b)*Ap + a]
 *   order AB (B innermost): codes[((h*d3 + w)*Ap + a)*Bp + b]
 * 4-bit codes are packed two per byte, even element in the low nibble.
 *
 * Padded extents: only the innermost axis is padded, to a whole number of
 * 16-byte rows (16 FP8 codes or 32 FP4 codes), so that every row starts on a
 * 16-byte boundary; the other axis keeps its size.  A block that runs past
 * the end of its axis is short: it covers only the real elements (zeros never
 * raise a block's absolute maximum, so this equals zero-padding the block).
 * Scales (one byte per block; nb(x) = ceil(x / 32)):
 *   A32 : scales[(pix*Bp + b)*nb(Ap) + a/32]
 *   B32 : scales[(pix*nb(Bp) + b/32)*Ap + a]
 *   SQ32: scales[(pix*nb(Bp) + b/32)*nb(Ap) + a/32]
 */
static int64_t nb32(int64_t x) { return (x + 31) / 32; }

void oracle_padded_extents(int fmt, int order, int64_t A, int64_t B, int64_t *Ap, int64_t *Bp)
{
    int64_t row = fmt_bits(fmt) == 4 ? 32 : 16;      /* elements per 16 bytes */
    *Ap = (order == OR_ORDER_BA) ? (A + row - 1) / row * row : A;
    *Bp = (order == OR_ORDER_AB) ? (B + row - 1) / row * row : B;
}

int64_t oracle_codes_bytes(int fmt, int order, int64_t d0, int64_t d1, int64_t d2, int64_t d3)
{
    int64_t Ap, Bp;
    oracle_padded_extents(fmt, order, d1, d0, &Ap, &Bp);
    int64_t n = d2 * d3 * Ap * Bp;
    return fmt_bits(fmt) == 4 ? n / 2 : n;
}

int64_t oracle_scales_bytes(int fmt, int block, int order, int64_t d0, int64_t d1, int64_t d2, int64_t d3)
{
    int64_t Ap, Bp;
    oracle_padded_extents(fmt, order, d1, d0, &Ap, &Bp);
    int64_t pix = d2 * d3;
    if (block == OR_A32) return pix * Bp * nb32(Ap);
    if (block == OR_B32) return pix * nb32(Bp) * Ap;
    return pix * nb32(Bp) * nb32(Ap);
}

static int64_t code_index(int order, int64_t pix, int64_t b, int64_t a, int64_t Ap, int64_t Bp)
{
    return order == OR_ORDER_BA ? (pix * Bp + b) * Ap + a : (pix * Ap + a) * Bp + b;
}

static int64_t scale_index(int block, int64_t pix, int64_t b, int64_t a, int64_t Ap, int64_t Bp)
{
    if (block == OR_A32) return (pix * Bp + b) * nb32(Ap) + a / 32;
    if (block == OR_B32) return (pix * nb32(Bp) + b / 32) * Ap + a;
    return (pix * nb32(Bp) + b / 32) * nb32(Ap) + a / 32;
}

static void put_code(uint8_t *codes, int fmt, int64_t idx, int code)
{
    if (fmt_bits(fmt) == 8) { codes[idx] = (uint8_t)code; return; }
    uint8_t *p = &codes[idx / 2];
    if (idx % 2 == 0) *p = (uint8_t)((*p & 0xF0) | (code & 0xF));
    else              *p = (uint8_t)((*p & 0x0F) | ((code & 0xF) << 4));
}

static int get_code(const uint8_t *codes, int fmt, int64_t idx)
{
    if (fmt_bits(fmt) == 8) return codes[idx];
    uint8_t v = codes[idx / 2];
    return idx % 2 == 0 ? (v & 0xF) : (v >> 4);
}

/* Source element (b, a, h, w), zero outside the real extents (padding). */
static double src_at(const float *src, int64_t d0, int64_t d1, const int64_t *st,
                     int64_t b, int64_t a, int64_t h, int64_t w)
{
    if (b >= d0 || a >= d1) return 0.0;
    return (double)src[b * st[0] + a * st[1] + h * st[2] + w * st[3]];
}

/* MX quantization of one tensor (paper, section III-A with the OCP MX block
 * scale; blocks oriented as in section IV-B).  Every block is visited once:
 * its amax gives the scale, then each element is encoded at that scale. */
void oracle_quantize(const float *src, int64_t d0, int64_t d1, int64_t d2, int64_t d3,
                     const int64_t *strides, int fmt, int block, int order,
                     uint8_t *codes, uint8_t *scales)
{
    int64_t Ap, Bp;
    oracle_padded_extents(fmt, order, d1, d0, &Ap, &Bp);
    int64_t nbytes = oracle_codes_bytes(fmt, order, d0, d1, d2, d3);
    memset(codes, 0, (size_t)nbytes);
    /* block extent along B and along A */
    int64_t eb = (block == OR_A32) ? 1 : 32;
    int64_t ea = (block == OR_B32) ? 1 : 32;
    int64_t npix = d2 * d3;
#pragma omp parallel for schedule(static)
    for (int64_t pix = 0; pix < npix; ++pix) {
        int64_t h = pix / d3, w = pix % d3;
        for (int64_t b0 = 0; b0 < Bp; b0 += eb)
            for (int64_t a0 = 0; a0 < Ap; a0 += ea) {
                int64_t b1 = b0 + eb < Bp ? b0 + eb : Bp, a1 = a0 + ea < Ap ? a0 + ea : Ap;
                double amax = 0.0;
                for (int64_t b = b0; b < b1; ++b)
                    for (int64_t a = a0; a < a1; ++a) {
                        double x = fabs(src_at(src, d0, d1, strides, b, a, h, w));
                        if (x > amax || x != x) amax = x;
                    }
                int sc = oracle_scale_code(fmt, amax);
                scales[scale_index(block, pix, b0, a0, Ap, Bp)] = (uint8_t)sc;
                double inv = ldexp(1.0, 127 - sc);       /* 2^-e, exact */
                for (int64_t b = b0; b < b1; ++b)
                    for (int64_t a = a0; a < a1; ++a) {
                        double x = src_at(src, d0, d1, strides, b, a, h, w);
                        int code = oracle_encode(fmt, x * inv);
                        put_code(codes, fmt, code_index(order, pix, b, a, Ap, Bp), code);
                    }
            }
    }
}

/* ------------------------------------------------------------------------ */
/* Stochastic rounding (paper, section III-A, Eq. 6 and the text after it:    */
/* gradients are rounded stochastically, activations and weights to nearest) */
/* ------------------------------------------------------------------------ */
/* Philox4x64-10, the counter-based generator of Salmon, Moraes, Dror and
 * Shaw ("Parallel random numbers: as easy as 1, 2, 3", SC 2011): ten rounds
 * of two 64x64->128-bit multiplications with the published multipliers
 * and Weyl key increments.  out[i] is word i of the block for (ctr, key). */
static void mulhilo64(uint64_t a, uint64_t b, uint64_t *hi, uint64_t *lo)
{
    unsigned __int128 p = (unsigned __int128)a * b;
    *hi = (uint64_t)(p >> 64);
    *lo = (uint64_t)p;
}

void oracle_philox4x64(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4])
{
    uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) { k0 += 0x9E3779B97F4A7C15ull; k1 += 0xBB67AE8584CAA73Bull; }
        uint64_t h0, l0, h1, l1;
        mulhilo64(0xD2E7470EE14C6C93ull, c0, &h0, &l0);
        mulhilo64(0xCA5A826395121157ull, c2, &h1, &l1);
        uint64_t n0 = h1 ^ c1 ^ k0, n1 = l1, n2 = h0 ^ c3 ^ k1, n3 = l0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 16 random bits of element (pix, b, a) of a tensor with extents
 * (d0 = B, d1 = A): element index i = ((pix*B + b)*A16 + a) with A16 = A
 * rounded up to 16, Philox block i / 16 (counter (i / 16, offset, 0, 0),
 * key (seed, 0)), bits 16*(j % 4) .. +15 of word j / 4, j = i % 16. */
uint32_t oracle_sr_bits(uint64_t seed, uint64_t offset, int64_t B, int64_t A, int64_t pix, int64_t b, int64_t a)
{
    int64_t A16 = (A + 15) / 16 * 16;
    uint64_t i = (uint64_t)((pix * B + b) * A16 + a);
    uint64_t ctr[4] = {i / 16, offset, 0, 0}, key[2] = {seed, 0}, out[4];
    oracle_philox4x64(ctr, key, out);
    int j = (int)(i % 16);
    return (uint32_t)((out[j / 4] >> (16 * (j % 4))) & 0xFFFFu);
}

/* Stochastic rounding of a real value v to the element format with 16
 * uniform random bits r: |v| lies between neighbouring finite magnitudes
 * lo <= |v| < hi; with f = (|v| - lo) / (hi - lo), the magnitude becomes hi
 * when r < f * 2^16 and lo otherwise (so hi with probability f, up to
 * 2^-16).  Magnitudes at or beyond the largest finite value saturate to it;
 * the sign is kept (also for zero). */
int oracle_encode_sr(int fmt, double v, uint32_t r)
{
    const or_table *t = table_of(fmt);
    int nb = fmt_bits(fmt);
    if (v != v) return fmt == OR_E2M1 ? 0x7 : 0x7F;
    int sign = signbit(v) ? 1 : 0;
    double a = fabs(v);
    int code;
    if (a >= t->val[t->n - 1]) {
        code = t->code[t->n - 1];
    } else {
        int lo = 0, hi = t->n - 1;                    /* val[lo] <= a < val[hi] */
        while (hi - lo > 1) {
            int mid = (lo + hi) / 2;
            if (t->val[mid] <= a) lo = mid; else hi = mid;
        }
        double f = (a - t->val[lo]) / (t->val[hi] - t->val[lo]);
        code = ((double)r < f * 65536.0) ? t->code[hi] : t->code[lo];
    }
    return (sign << (nb - 1)) | code;
}

/* MX quantization with stochastic rounding of the elements: the blocks and
 * E8M0 scales are those of oracle_quantize (section III-A with the OCP
 * scale), each element x*2^-e is rounded by oracle_encode_sr with the bits
 * oracle_sr_bits gives for its position. */
void oracle_quantize_sr(const float *src, int64_t d0, int64_t d1, int64_t d2, int64_t d3,
                        const int64_t *strides, int fmt, int block, int order,
                        uint64_t seed, uint64_t offset, uint8_t *codes, uint8_t *scales)
{
    int64_t Ap, Bp;
    oracle_padded_extents(fmt, order, d1, d0, &Ap, &Bp);
    int64_t nbytes = oracle_codes_bytes(fmt, order, d0, d1, d2, d3);
    memset(codes, 0, (size_t)nbytes);
    int64_t eb = (block == OR_A32) ? 1 : 32;
    int64_t ea = (block == OR_B32) ? 1 : 32;
    int64_t npix = d2 * d3;
#pragma omp parallel for schedule(static)
    for (int64_t pix = 0; pix < npix; ++pix) {
        int64_t h = pix / d3, w = pix % d3;
        for (int64_t b0 = 0; b0 < Bp; b0 += eb)
            for (int64_t a0 = 0; a0 < Ap; a0 += ea) {
                int64_t b1 = b0 + eb < Bp ? b0 + eb : Bp, a1 = a0 + ea < Ap ? a0 + ea : Ap;
                double amax = 0.0;
                for (int64_t b = b0; b < b1; ++b)
                    for (int64_t a = a0; a < a1; ++a) {
                        double x = fabs(src_at(src, d0, d1, strides, b, a, h, w));
                        if (x > amax || x != x) amax = x;
                    }
                int sc = oracle_scale_code(fmt, amax);
                scales[scale_index(block, pix, b0, a0, Ap, Bp)] = (uint8_t)sc;
                double inv = ldexp(1.0, 127 - sc);
                for (int64_t b = b0; b < b1; ++b)
                    for (int64_t a = a0; a < a1; ++a) {
                        if (b >= d0 || a >= d1) continue;     /* padding stays +0 */
                        double x = src_at(src, d0, d1, strides, b, a, h, w);
                        uint32_t r = oracle_sr_bits(seed, offset, d0, d1, pix, b, a);
                        int code = oracle_encode_sr(fmt, x * inv, r);
                        put_code(codes, fmt, code_index(order, pix, b, a, Ap, Bp), code);
                    }
            }
    }
}

/* ------------------------------------------------------------------------ */
/* NVFP4: the format of the paper's own experiments (section III-A,        */
/* Eq. 4-6): a per-tensor FP32 scale, an E4M3 scale per block of 16,        */
/* E2M1 elements                                                             */
/* ------------------------------------------------------------------------ */
/* Blocks of 16: along the A-axis (NV_A16), along the B-axis (NV_B16), or a
 * 16x16 square over (B, A) (NV_SQ16).  The pages give the steps as real
 * formulas; they are evaluated here in IEEE fp32, one rounding per step in
 * the order the equations write them (the precision the CUDA kernel decides
 * the codes in):
 *   Eq. 4  T  = max|X| / (448 * 6)
 *   Eq. 5  Bs = CastE4M3( max|X_i| / (T * 6) )      round to nearest even
 *   Eq. 6  q  = Round( x / (Bs * T) )               E2M1, nearest even, saturating
 * A block whose scale is 0 (or a tensor whose maximum is 0) gets zero codes
 * (x * 0, so the sign of zero is kept).  Layout: the E2M1 codes as in
 * oracle_quantize; one E4M3 scale byte per block:
 *   NV_A16 : scales[(pix*Bp + b)*nb16(Ap) + a/16]
 *   NV_B16 : scales[(pix*nb16(Bp) + b/16)*Ap + a]
 *   NV_SQ16: scales[(pix*nb16(Bp) + b/16)*nb16(Ap) + a/16] */
enum { NV_A16 = 0, NV_B16 = 1, NV_SQ16 = 2 };
static int64_t nb16(int64_t x) { return (x + 15) / 16; }

int64_t oracle_nvfp4_scales_bytes(int block, int order, int64_t d0, int64_t d1, int64_t d2, int64_t d3)
{
    int64_t Ap, Bp;
    oracle_padded_extents(OR_E2M1, order, d1, d0, &Ap, &Bp);
    int64_t pix = d2 * d3;
    if (block == NV_A16) return pix * Bp * nb16(Ap);
    if (block == NV_B16) return pix * nb16(Bp) * Ap;
    return pix * nb16(Bp) * nb16(Ap);
}

static int64_t nv_scale_index(int block, int64_t pix, int64_t b, int64_t a, int64_t Ap, int64_t Bp)
{
    if (block == NV_A16) return (pix * Bp + b) * nb16(Ap) + a / 16;
    if (block == NV_B16) return (pix * nb16(Bp) + b / 16) * Ap + a;
    return (pix * nb16(Bp) + b / 16) * nb16(Ap) + a / 16;
}

void oracle_quantize_nvfp4(const float *src, int64_t d0, int64_t d1, int64_t d2, int64_t d3,
                           const int64_t *strides, int block, int order,
                           uint8_t *codes, uint8_t *scales, float *tscale)
{
    int64_t Ap, Bp;
    oracle_padded_extents(OR_E2M1, order, d1, d0, &Ap, &Bp);
    memset(codes, 0, (size_t)oracle_codes_bytes(OR_E2M1, order, d0, d1, d2, d3));
    float amax = 0.0f;
    for (int64_t b = 0; b < d0; ++b)
        for (int64_t a = 0; a < d1; ++a)
            for (int64_t h = 0; h < d2; ++h)
                for (int64_t w = 0; w < d3; ++w) {
                    float x = fabsf(src[b * strides[0] + a * strides[1] + h * strides[2] + w * strides[3]]);
                    if (x > amax) amax = x;
                }
    const float T = amax / 2688.0f;                       /* Eq. 4: 448 * 6 */
    *tscale = T;
    const float d = T * 6.0f;
    int64_t eb = (block == NV_A16) ? 1 : 16;
    int64_t ea = (block == NV_B16) ? 1 : 16;
    int64_t npix = d2 * d3;
#pragma omp parallel for schedule(static)
    for (int64_t pix = 0; pix < npix; ++pix) {
        int64_t h = pix / d3, w = pix % d3;
        for (int64_t b0 = 0; b0 < Bp; b0 += eb)
            for (int64_t a0 = 0; a0 < Ap; a0 += ea) {
                int64_t b1 = b0 + eb < Bp ? b0 + eb : Bp, a1 = a0 + ea < Ap ? a0 + ea : Ap;
                float bmax = 0.0f;
                for (int64_t b = b0; b < b1; ++b)
                    for (int64_t a = a0; a < a1; ++a) {
                        float x = fabsf((float)src_at(src, d0, d1, strides, b, a, h, w));
                        if (x > bmax) bmax = x;
                    }
                const float q = T > 0.0f ? bmax / d : 0.0f;                     /* Eq. 5 */
                const int sc = oracle_encode(OR_E4M3, (double)q);
                scales[nv_scale_index(block, pix, b0, a0, Ap, Bp)] = (uint8_t)sc;
                int fin;
                const float Bs = (float)oracle_decode(OR_E4M3, sc, &fin);
                const float s = Bs * T;
                for (int64_t b = b0; b < b1; ++b)
                    for (int64_t a = a0; a < a1; ++a) {
                        if (b >= d0 || a >= d1) continue;
                        const float x = (float)src_at(src, d0, d1, strides, b, a, h, w);
                        const float v = s > 0.0f ? x / s : x * 0.0f;              /* Eq. 6 */
                        put_code(codes, OR_E2M1, code_index(order, pix, b, a, Ap, Bp), oracle_encode(OR_E2M1, (double)v));
                    }
            }
    }
}

/* Dense double tensor of an NVFP4 quantization: element value * Bs * T. */
void oracle_dequantize_nvfp4(const uint8_t *codes, const uint8_t *scales, float tscale, int64_t d0, int64_t d1,
                             int64_t d2, int64_t d3, int block, int order, double *out)
{
    int64_t Ap, Bp;
    oracle_padded_extents(OR_E2M1, order, d1, d0, &Ap, &Bp);
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < d0; ++b)
        for (int64_t a = 0; a < d1; ++a)
            for (int64_t h = 0; h < d2; ++h)
                for (int64_t w = 0; w < d3; ++w) {
                    int64_t pix = h * d3 + w;
                    int fin;
                    double v = oracle_decode(OR_E2M1, get_code(codes, OR_E2M1, code_index(order, pix, b, a, Ap, Bp)), &fin);
                    double bs = oracle_decode(OR_E4M3, scales[nv_scale_index(block, pix, b, a, Ap, Bp)], &fin);
                    out[((b * d1 + a) * d2 + h) * d3 + w] = v * bs * (double)tscale;
                }
}

/* Dequantize back to a dense double tensor [d0][d1][d2][d3]:
 * value = element value * 2^(scale - 127). */
void oracle_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t d0, int64_t d1,
                       int64_t d2, int64_t d3, int fmt, int block, int order, double *out)
{
    int64_t Ap, Bp;
    oracle_padded_extents(fmt, order, d1, d0, &Ap, &Bp);
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < d0; ++b)
        for (int64_t a = 0; a < d1; ++a)
            for (int64_t h = 0; h < d2; ++h)
                for (int64_t w = 0; w < d3; ++w) {
                    int64_t pix = h * d3 + w;
                    int fin;
                    double v = oracle_decode(fmt, get_code(codes, fmt, code_index(order, pix, b, a, Ap, Bp)), &fin);
                    int sc = scales[scale_index(block, pix, b, a, Ap, Bp)];
                    out[((b * d1 + a) * d2 + h) * d3 + w] = sc == 0xFF ? NAN : ldexp(v, sc - 127);
                }
}

/* ------------------------------------------------------------------------ */
/* im2col                                                                    */
/* ------------------------------------------------------------------------ */
/* Output spatial size with stride and zero padding (PyTorch semantics). */
static int64_t out_size(int64_t in, int64_t k, int64_t s, int64_t p) { return (in + 2 * p - k) / s + 1; }

/* Naive im2col of fp32 X [N][Cin][Hin][Win] (paper, section II-C1), emitted in
 * the channel-batch-first row order (K_h K_w C_in) of section IV-B, as a dense
 * tensor Xe [N][Kh*Kw*Cin][Hout][Wout]: channel (r*Kw + s)*Cin + c of output
 * pixel (p, q) is X[n][c][p*sh + r - ph][q*sw + s - pw], or 0 in the padding. */
void oracle_im2col_fp32(const float *X, int64_t N, int64_t Cin, int64_t Hin, int64_t Win,
                        int64_t Kh, int64_t Kw, int64_t sh, int64_t sw, int64_t ph, int64_t pw,
                        float *Xe)
{
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
    int64_t CE = Kh * Kw * Cin;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t r = 0; r < Kh; ++r)
            for (int64_t s = 0; s < Kw; ++s)
                for (int64_t c = 0; c < Cin; ++c)
                    for (int64_t p = 0; p < Ho; ++p)
                        for (int64_t q = 0; q < Wo; ++q) {
                            int64_t h = p * sh + r - ph, w = q * sw + s - pw;
                            float v = 0.0f;
                            if (h >= 0 && h < Hin && w >= 0 && w < Win)
                                v = X[((n * Cin + c) * Hin + h) * Win + w];
                            Xe[((n * CE + (r * Kw + s) * Cin + c) * Ho + p) * Wo + q] = v;
                        }
}

/* Channel-batch-first im2col on already-quantized codes and scales (paper,
 * section IV-A).  The source is X quantized in the layout above (B = N,
 * A = C_in, spatial Hin x Win, padded A extent Ap).  The result is the same
 * layout for the expanded tensor: spatial Hout x Wout, B = N, A-axis
 * (r, s, c) of extent Kh*Kw*Ap with c fastest.  Positions in the padding get
 * code +0 and, for blocks wholly in the padding, scale 0x00. */
void oracle_im2col_cbf(const uint8_t *codes, const uint8_t *scales,
                       int64_t N, int64_t Cin, int64_t Hin, int64_t Win,
                       int64_t Kh, int64_t Kw, int64_t sh, int64_t sw, int64_t ph, int64_t pw,
                       int fmt, int block, int order, uint8_t *codes_out, uint8_t *scales_out)
{
    int64_t Ap, Bp;
    oracle_padded_extents(fmt, order, Cin, N, &Ap, &Bp);
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
    int64_t Ae = Kh * Kw * Ap;              /* expanded A extent: Ap per tap */
    int64_t nb = oracle_codes_bytes(fmt, order, Bp, Ae, Ho, Wo);
    memset(codes_out, 0, (size_t)nb);
    int64_t n_sb = (block == OR_A32) ? Bp : nb32(Bp);       /* scale rows per pixel */
    int64_t n_sa = (block == OR_B32) ? Ap : nb32(Ap);       /* scale cols per tap */
    int64_t n_sa_e = Kh * Kw * n_sa;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < Ho; ++p)
        for (int64_t q = 0; q < Wo; ++q)
            for (int64_t r = 0; r < Kh; ++r)
                for (int64_t s = 0; s < Kw; ++s) {
                    int64_t h = p * sh + r - ph, w = q * sw + s - pw;
                    int inside = (h >= 0 && h < Hin && w >= 0 && w < Win);
                    int64_t pix_o = p * Wo + q, pix_i = inside ? h * Win + w : 0;
                    int64_t a_off = (r * Kw + s) * Ap;
                    for (int64_t b = 0; b < Bp; ++b)
                        for (int64_t c = 0; c < Ap; ++c) {
                            int code = inside ? get_code(codes, fmt, code_index(order, pix_i, b, c, Ap, Bp)) : 0;
                            put_code(codes_out, fmt, code_index(order, pix_o, b, a_off + c, Ae, Bp), code);
                        }
                    for (int64_t ib = 0; ib < n_sb; ++ib)
                        for (int64_t ia = 0; ia < n_sa; ++ia) {
                            uint8_t sc = inside ? scales[(pix_i * n_sb + ib) * n_sa + ia] : 0;
                            int64_t ia_e = (r * Kw + s) * n_sa + ia;
                            scales_out[(pix_o * n_sb + ib) * n_sa_e + ia_e] = sc;
                        }
                }
}

/* ------------------------------------------------------------------------ */
/* Direct convolutions in double (paper, section II-A, Eq. 1-3)              */
/* ------------------------------------------------------------------------ */
/* Forward, Eq. 1: Y[n][k][p][q] = sum_{c,r,s} W[k][c][r][s] * X[n][c][p*sh+r-ph][q*sw+s-pw]. */
void oracle_conv_fwd(const double *X, const double *W, int64_t N, int64_t Cin, int64_t Hin, int64_t Win,
                     int64_t Cout, int64_t Kh, int64_t Kw, int64_t sh, int64_t sw, int64_t ph, int64_t pw,
                     double *Y, double *Yabs)
{
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < Cout; ++k)
            for (int64_t p = 0; p < Ho; ++p)
                for (int64_t q = 0; q < Wo; ++q) {
                    double acc = 0.0, aabs = 0.0;
                    for (int64_t c = 0; c < Cin; ++c)
                        for (int64_t r = 0; r < Kh; ++r)
                            for (int64_t s = 0; s < Kw; ++s) {
                                int64_t h = p * sh + r - ph, w = q * sw + s - pw;
                                if (h < 0 || h >= Hin || w < 0 || w >= Win) continue;
                                double t = W[((k * Cin + c) * Kh + r) * Kw + s] * X[((n * Cin + c) * Hin + h) * Win + w];
                                acc += t;
                                aabs += fabs(t);
                            }
                    int64_t o = ((n * Cout + k) * Ho + p) * Wo + q;
                    Y[o] = acc;
                    if (Yabs) Yabs[o] = aabs;
                }
}

/* Input gradient, Eq. 2 (the exact derivative of the forward above):
 * G_X[n][c][h][w] = sum over (k, r, s) with h = p*sh + r - ph and
 * w = q*sw + s - pw for an output position (p, q) of W[k][c][r][s] * G_Y[n][k][p][q]. */
void oracle_conv_dgrad(const double *W, const double *GY, int64_t N, int64_t Cin, int64_t Hin, int64_t Win,
                       int64_t Cout, int64_t Kh, int64_t Kw, int64_t sh, int64_t sw, int64_t ph, int64_t pw,
                       double *GX, double *GXabs)
{
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t c = 0; c < Cin; ++c)
            for (int64_t h = 0; h < Hin; ++h)
                for (int64_t w = 0; w < Win; ++w) {
                    double acc = 0.0, aabs = 0.0;
                    for (int64_t k = 0; k < Cout; ++k)
                        for (int64_t r = 0; r < Kh; ++r)
                            for (int64_t s = 0; s < Kw; ++s) {
                                int64_t hp = h + ph - r, wq = w + pw - s;
                                if (hp < 0 || wq < 0 || hp % sh != 0 || wq % sw != 0) continue;
                                int64_t p = hp / sh, q = wq / sw;
                                if (p >= Ho || q >= Wo) continue;
                                double t = W[((k * Cin + c) * Kh + r) * Kw + s] * GY[((n * Cout + k) * Ho + p) * Wo + q];
                                acc += t;
                                aabs += fabs(t);
                            }
                    int64_t o = ((n * Cin + c) * Hin + h) * Win + w;
                    GX[o] = acc;
                    if (GXabs) GXabs[o] = aabs;
                }
}

/* Weight gradient, Eq. 3: G_W[k][c][r][s] = sum_{n,p,q} G_Y[n][k][p][q] * X[n][c][p*sh+r-ph][q*sw+s-pw]. */
void oracle_conv_wgrad(const double *GY, const double *X, int64_t N, int64_t Cin, int64_t Hin, int64_t Win,
                       int64_t Cout, int64_t Kh, int64_t Kw, int64_t sh, int64_t sw, int64_t ph, int64_t pw,
                       double *GW, double *GWabs)
{
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t k = 0; k < Cout; ++k)
        for (int64_t c = 0; c < Cin; ++c)
            for (int64_t r = 0; r < Kh; ++r)
                for (int64_t s = 0; s < Kw; ++s) {
                    double acc = 0.0, aabs = 0.0;
                    for (int64_t n = 0; n < N; ++n)
                        for (int64_t p = 0; p < Ho; ++p)
                            for (int64_t q = 0; q < Wo; ++q) {
                                int64_t h = p * sh + r - ph, w = q * sw + s - pw;
                                if (h < 0 || h >= Hin || w < 0 || w >= Win) continue;
                                double t = GY[((n * Cout + k) * Ho + p) * Wo + q] * X[((n * Cin + c) * Hin + h) * Win + w];
                                acc += t;
                                aabs += fabs(t);
                            }
                    int64_t o = ((k * Cin + c) * Kh + r) * Kw + s;
                    GW[o] = acc;
                    if (GWabs) GWabs[o] = aabs;
                }
}

/* Selected outputs only: the same sums as above evaluated at a list of flat
 * output indices (used to check very large problems on sampled positions). */
void oracle_conv_fwd_at(const double *X, const double *W, int64_t N, int64_t Cin, int64_t Hin, int64_t Win,
                        int64_t Cout, int64_t Kh, int64_t Kw, int64_t sh, int64_t sw, int64_t ph, int64_t pw,
                        const int64_t *idx, int64_t nidx, double *val, double *vabs)
{
    (void)N;
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nidx; ++i) {
        int64_t o = idx[i];
        int64_t q = o % Wo, p = (o / Wo) % Ho, k = (o / (Wo * Ho)) % Cout, n = o / (Wo * Ho * Cout);
        double acc = 0.0, aabs = 0.0;
        for (int64_t c = 0; c < Cin; ++c)
            for (int64_t r = 0; r < Kh; ++r)
                for (int64_t s = 0; s < Kw; ++s) {
                    int64_t h = p * sh + r - ph, w = q * sw + s - pw;
                    if (h < 0 || h >= Hin || w < 0 || w >= Win) continue;
                    double t = W[((k * Cin + c) * Kh + r) * Kw + s] * X[((n * Cin + c) * Hin + h) * Win + w];
                    acc += t;
                    aabs += fabs(t);
                }
        val[i] = acc;
        vabs[i] = aabs;
    }
}

void oracle_conv_dgrad_at(const double *W, const double *GY, int64_t N, int64_t Cin, int64_t Hin, int64_t Win,
                          int64_t Cout, int64_t Kh, int64_t Kw, int64_t sh, int64_t sw, int64_t ph, int64_t pw,
                          const int64_t *idx, int64_t nidx, double *val, double *vabs)
{
    (void)N;
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nidx; ++i) {
        int64_t o = idx[i];
        int64_t w = o % Win, h = (o / Win) % Hin, c = (o / (Win * Hin)) % Cin, n = o / (Win * Hin * Cin);
        double acc = 0.0, aabs = 0.0;
        for (int64_t k = 0; k < Cout; ++k)
            for (int64_t r = 0; r < Kh; ++r)
                for (int64_t s = 0; s < Kw; ++s) {
                    int64_t hp = h + ph - r, wq = w + pw - s;
                    if (hp < 0 || wq < 0 || hp % sh != 0 || wq % sw != 0) continue;
                    int64_t p = hp / sh, q = wq / sw;
                    if (p >= Ho || q >= Wo) continue;
                    double t = W[((k * Cin + c) * Kh + r) * Kw + s] * GY[((n * Cout + k) * Ho + p) * Wo + q];
                    acc += t;
                    aabs += fabs(t);
                }
        val[i] = acc;
        vabs[i] = aabs;
    }
}

void oracle_conv_wgrad_at(const double *GY, const double *X, int64_t N, int64_t Cin, int64_t Hin, int64_t Win,
                          int64_t Cout, int64_t Kh, int64_t Kw, int64_t sh, int64_t sw, int64_t ph, int64_t pw,
                          const int64_t *idx, int64_t nidx, double *val, double *vabs)
{
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nidx; ++i) {
        int64_t o = idx[i];
        int64_t s = o % Kw, r = (o / Kw) % Kh, c = (o / (Kw * Kh)) % Cin, k = o / (Kw * Kh * Cin);
        double acc = 0.0, aabs = 0.0;
        for (int64_t n = 0; n < N; ++n)
            for (int64_t p = 0; p < Ho; ++p)
                for (int64_t q = 0; q < Wo; ++q) {
                    int64_t h = p * sh + r - ph, w = q * sw + s - pw;
                    if (h < 0 || h >= Hin || w < 0 || w >= Win) continue;
                    double t = GY[((n * Cout + k) * Ho + p) * Wo + q] * X[((n * Cin + c) * Hin + h) * Win + w];
                    acc += t;
                    aabs += fabs(t);
                }
        val[i] = acc;
        vabs[i] = aabs;
    }
}

/* ------------------------------------------------------------------------ */
/* Quantization-count and stored-bytes model (paper, section IV-C, Table I)  */
/* ------------------------------------------------------------------------ */
/* counts[n][c][h][w] = number of entries of the im2col matrix X' that are the
 * source element X[n][c][h][w] (enumerated from the im2col index map).  A
 * method that quantizes X' once (square blocks, Cuyckens et al.) quantizes
 * each source element that many times; one that quantizes it once per
 * direction (DaCapo line blocks) twice that; MicroQonv quantizes X before the
 * expansion, so once.  Returns the number of entries of X' (padding included). */
int64_t oracle_im2col_counts(int64_t N, int64_t Cin, int64_t Hin, int64_t Win, int64_t Kh, int64_t Kw,
                             int64_t sh, int64_t sw, int64_t ph, int64_t pw, int32_t *counts)
{
    int64_t Ho = out_size(Hin, Kh, sh, ph), Wo = out_size(Win, Kw, sw, pw);
    memset(counts, 0, sizeof(int32_t) * (size_t)(N * Cin * Hin * Win));
    int64_t entries = 0;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t c = 0; c < Cin; ++c)
            for (int64_t r = 0; r < Kh; ++r)
                for (int64_t s = 0; s < Kw; ++s)
                    for (int64_t p = 0; p < Ho; ++p)
                        for (int64_t q = 0; q < Wo; ++q) {
                            ++entries;
                            int64_t h = p * sh + r - ph, w = q * sw + s - pw;
                            if (h < 0 || h >= Hin || w < 0 || w >= Win) continue;
                            counts[((n * Cin + c) * Hin + h) * Win + w]++;
                        }
    return entries;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
