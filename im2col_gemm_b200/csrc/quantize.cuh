// quantize.cuh -- single-pass OCP-MX quantization into the channel-batch-first
// layout (MicroQonv paper, arXiv:2609.28358: section III-A for the
// microscaling steps with the OCP E8M0 shared scale, section IV-B for the
// quantization directions, section IV-A / Fig. 3 for the layout).
//
// One CTA (8 warps) handles a tile of 32 or 64 spatial positions x OT x IT of
// the (B, A) plane, where i is the primary order's innermost axis (IT = 32,
// or 16 when that axis has at most 16 FP8 elements) and o the other axis
// (OT = 32, or 16 when it has at most 16 elements; the spare warps then take
// a second group of 32 positions).  Lane = spatial position, so fp32 reads
// along the flattened H*W axis of an NCHW source are coalesced.  A thread
// owns 4 o-rows x IT values and holds one row at a time.  Blocks along i
// take their maximum in registers; blocks along o and 32x32 squares first
// reduce through shared-memory atomics (phase 1) and the rows are read again,
// mostly from L2, to convert (phase 2).  Conversion is cvt.rn.satfinite; the
// primary rows are stored directly, the optional second code order goes
// through a padded shared-memory transpose.
#pragma once

#include "common.cuh"

namespace mqc {

struct QuantParams {
    const float *src;
    int64_t sb, sa, sh, sw;     // element strides of the B, A, H, W axes
    int32_t B, A, H, W;         // real extents
    int32_t npix;               // H * W
    // primary order: codes[(pix*O + o)*I1 + i]   (I1 = padded innermost extent)
    uint8_t *codes;
    int32_t I1;
    // optional second order: codes_alt[(pix*I + i)*O2 + o]   (O2 padded)
    uint8_t *codes_alt;
    int32_t O2;
    uint8_t *scales;
    int32_t Ap1, Bp1;           // primary padded extents, for the scale layout
    int32_t fmt;                // 0 E4M3, 1 E5M2, 2 E2M1
    int32_t emax;               // emax_elem of fmt
    int32_t OT;                 // tile extent along o (16 or 32)
    int32_t nPT, nOT, nIT;      // tile counts along positions, o and i
    int32_t I, O;               // real extents along i and o
};

// E8M0 code of a block with absolute maximum `amax`: e = floor(log2 amax) -
// emax, clamped below at -127 (so zero and subnormal maxima give 0x00); a
// non-finite maximum gives 0xFF.
__device__ __forceinline__ uint32_t e8m0_code(float amax, int emax) {
    const uint32_t bits = __float_as_uint(amax);
    if (bits >= 0x7F800000u) return 0xFFu;
    const int ex = static_cast<int>(bits >> 23);
    const int c = ex - emax;
    return (ex == 0 || c < 0) ? 0u : static_cast<uint32_t>(c);
}

// 2^-e for the scale code (an exact power of two, always a normal float).
__device__ __forceinline__ float e8m0_inv(uint32_t code) {
    if (code == 0xFFu) return __uint_as_float(0x00400000u);   // 2^-128
    return __uint_as_float((254u - code) << 23);
}

// Two codes from two fp32 values, round-to-nearest-even with saturation to
// the largest finite value; `lo` lands in the low byte / nibble.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t cvt_e5m2x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// FMT: 0 E4M3, 1 E5M2, 2 E2M1.
template <int FMT>
__device__ __forceinline__ uint32_t cvt_pair(float lo, float hi) {
    if (FMT == 0) return cvt_e4m3x2(lo, hi);
    if (FMT == 1) return cvt_e5m2x2(lo, hi);
    return cvt_e2m1x2(lo, hi);
}

enum QuantBlock : int { kAlongI = 0, kAlongO = 1, kSquare = 2 };

// MAP_A: the i axis is A (primary order BA); otherwise it is B (order AB).
// BLK: direction of the blocks relative to (i, o).  IT: 32 or 16 (FP8 only).
// The work of one CTA (256 threads) on tile `t` of the tensor p.
template <bool MAP_A, int BLK, int FMT, int IT, bool DUAL>
__device__ __forceinline__ void quantize_tile(const QuantParams &p, int t) {
    constexpr int OJ = 4;                             // o-rows per thread
    constexpr bool FP4 = FMT == 2;
    constexpr int RB = FP4 ? IT / 2 : IT;             // bytes of one 32- or 16-code row
    __shared__ float s_amax[2 * IT * 32];
    __shared__ uint32_t s_alt[64 * 129];              // >= positions x (IT*OT/4 + 1) words

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int wpg = p.OT / OJ;                        // warps per position group (4 or 8)
    const int grp = warp / wpg;
    const int wo = warp % wpg;
    const int gsize = 8 / wpg;                        // position groups per CTA (2 or 1)

    const int pT = t % p.nPT;
    t /= p.nPT;
    const int oT = t % p.nOT;
    const int iT = t / p.nOT;

    const int pix = (pT * gsize + grp) * 32 + lane;
    const bool pix_ok = pix < p.npix;
    const int h = pix_ok ? pix / p.W : 0;
    const int w = pix_ok ? pix % p.W : 0;
    const int o0 = oT * p.OT + wo * OJ;
    const int i0 = iT * IT;

    if (BLK != kAlongI) {
        for (int k = threadIdx.x; k < 2 * IT * 32; k += 256) s_amax[k] = 0.0f;
    }

    const float *base = p.src + static_cast<int64_t>(h) * p.sh + static_cast<int64_t>(w) * p.sw;
    const int64_t so = MAP_A ? p.sb : p.sa, si = MAP_A ? p.sa : p.sb;
    auto load_row = [&](int j, float (&r)[IT]) {
        const bool row_ok = pix_ok && (o0 + j) < p.O;
        const float *rp = base + static_cast<int64_t>(o0 + j) * so + static_cast<int64_t>(i0) * si;
#pragma unroll
        for (int k = 0; k < IT; ++k) r[k] = (row_ok && i0 + k < p.I) ? __ldg(rp + k * si) : 0.0f;
    };

    // ---- phase 1: maxima of blocks that span several threads (the rows are
    // read again in phase 2, mostly from L2, so a thread holds one row at a time)
    if (BLK != kAlongI) {
        __syncthreads();                              // s_amax cleared
        if (BLK == kAlongO) {
            float m[IT];
#pragma unroll
            for (int k = 0; k < IT; ++k) m[k] = 0.0f;
#pragma unroll 1
            for (int j = 0; j < OJ; ++j) {
                float r[IT];
                load_row(j, r);
#pragma unroll
                for (int k = 0; k < IT; ++k) m[k] = fmaxf(m[k], fabsf(r[k]));
            }
            float *am = s_amax + grp * IT * 32;
#pragma unroll
            for (int k = 0; k < IT; ++k) atomicMax(reinterpret_cast<int *>(am + k * 32 + lane), __float_as_int(m[k]));
        } else {
            float m = 0.0f;
#pragma unroll 1
            for (int j = 0; j < OJ; ++j) {
                float r[IT];
                load_row(j, r);
#pragma unroll
                for (int k = 0; k < IT; ++k) m = fmaxf(m, fabsf(r[k]));
            }
            atomicMax(reinterpret_cast<int *>(s_amax + grp * 32 + lane), __float_as_int(m));
        }
        __syncthreads();
    }

    // ---- scales of blocks spanning threads (layout of the primary order's padded extents)
    const int nbA = (p.Ap1 + 31) / 32, nbB = (p.Bp1 + 31) / 32;
    uint32_t code_sq = 0u;
    if (BLK == kSquare) {
        code_sq = e8m0_code(s_amax[grp * 32 + lane], p.emax);
        if (wo == 0 && pix_ok) {
            const int bT = MAP_A ? oT : iT, aT = MAP_A ? iT : oT;
            p.scales[(static_cast<int64_t>(pix) * nbB + bT) * nbA + aT] = code_sq;
        }
    } else if (BLK == kAlongO) {
        if (pix_ok) {
            const float *am = s_amax + grp * IT * 32;
            for (int k = wo; k < IT; k += wpg) {
                const int i = i0 + k;
                const uint32_t c = e8m0_code(am[k * 32 + lane], p.emax);
                if (MAP_A) {        // B32: block oT along b, column a = i
                    if (i < p.Ap1) p.scales[(static_cast<int64_t>(pix) * nbB + oT) * p.Ap1 + i] = c;
                } else {            // A32: row b = i, block oT along a
                    if (i < p.Bp1) p.scales[(static_cast<int64_t>(pix) * p.Bp1 + i) * nbA + oT] = c;
                }
            }
        }
    }
    const float inv_sq = BLK == kSquare ? e8m0_inv(code_sq) : 1.0f;
    float inv_k[BLK == kAlongO ? IT : 1];
    if (BLK == kAlongO) {
        const float *am = s_amax + grp * IT * 32;
#pragma unroll
        for (int k = 0; k < (BLK == kAlongO ? IT : 1); ++k) inv_k[k] = e8m0_inv(e8m0_code(am[k * 32 + lane], p.emax));
    }

    // ---- phase 2: per row, convert, store the primary row, collect the second order
    const int row_bytes = (p.I1 - i0) >= IT ? RB : (FP4 ? 0 : ((p.I1 - i0) >= 16 ? 16 : 0));
    uint32_t unit[DUAL ? IT : 1];
#pragma unroll
    for (int k = 0; k < (DUAL ? IT : 1); ++k) unit[k] = 0u;
#pragma unroll
    for (int j = 0; j < OJ; ++j) {
        float r[IT];
        load_row(j, r);
        const int o = o0 + j;
        float inv_row = inv_sq;
        if (BLK == kAlongI) {
            float m = 0.0f;
#pragma unroll
            for (int k = 0; k < IT; ++k) m = fmaxf(m, fabsf(r[k]));
            const uint32_t c = e8m0_code(m, p.emax);
            inv_row = e8m0_inv(c);
            if (pix_ok) {
                if (MAP_A) {        // A32: row b = o, block iT along a
                    if (o < p.Bp1) p.scales[(static_cast<int64_t>(pix) * p.Bp1 + o) * nbA + iT] = c;
                } else {            // B32: column a = o, block iT along b
                    if (o < p.Ap1) p.scales[(static_cast<int64_t>(pix) * nbB + iT) * p.Ap1 + o] = c;
                }
            }
        }
        uint32_t words[RB / 4];
#pragma unroll
        for (int q = 0; q < RB / 4; ++q) words[q] = 0u;
#pragma unroll
        for (int k = 0; k < IT; k += 2) {
            const float s0 = BLK == kAlongO ? inv_k[k % (BLK == kAlongO ? IT : 1)] : inv_row;
            const float s1 = BLK == kAlongO ? inv_k[(k + 1) % (BLK == kAlongO ? IT : 1)] : inv_row;
            const uint32_t pair = cvt_pair<FMT>(r[k] * s0, r[k + 1] * s1);
            if (FP4) {
                words[k / 8] |= pair << (4 * (k % 8));
                if (DUAL) {
                    unit[k] |= (pair & 0xFu) << (4 * j);
                    unit[k + 1] |= (pair >> 4) << (4 * j);
                }
            } else {
                words[k / 4] |= pair << (8 * (k % 4));
                if (DUAL) {
                    unit[k] |= (pair & 0xFFu) << (8 * j);
                    unit[k + 1] |= (pair >> 8) << (8 * j);
                }
            }
        }
        if (pix_ok && o < p.O && row_bytes > 0) {
            const int64_t off = (static_cast<int64_t>(pix) * p.O + o) * p.I1 + i0;
            uint4 *dst = reinterpret_cast<uint4 *>(p.codes + (FP4 ? off / 2 : off));
            dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
            if constexpr (RB == 32) {
                if (row_bytes == 32) dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
            }
        }
    }
    if (!DUAL) return;

    // units: FP8 -> a 32-bit word (4 codes), FP4 -> 16 bits (4 nibbles);
    // per position: IT rows of OT/4 units, plane pitch padded by one word
    const int upr = p.OT / OJ;                         // units per row
    const int plane = FP4 ? (IT * upr) / 2 + 1 : IT * upr + 1;   // words
    uint32_t *pl = s_alt + (grp * 32 + lane) * plane;
    if (FP4) {
        uint16_t *p16 = reinterpret_cast<uint16_t *>(pl);
#pragma unroll
        for (int k = 0; k < IT; ++k) p16[k * upr + wo] = static_cast<uint16_t>(unit[k]);
    } else {
#pragma unroll
        for (int k = 0; k < IT; ++k) pl[k * upr + wo] = unit[k];
    }
    __syncthreads();

    // rows (position, i) of the o-codes [oT*OT, oT*OT+OT) clipped to the padded O2
    const int o_base = oT * p.OT;
    const int full = FP4 ? p.OT / 2 : p.OT;            // bytes of one row of this tile
    const int alt_bytes = (p.O2 - o_base) >= p.OT ? full : (FP4 ? 0 : ((p.O2 - o_base) >= 16 ? 16 : 0));
    if (alt_bytes == 0) return;
    const int nch = alt_bytes / 16;
    const int npos = 32 * gsize;
    for (int id = threadIdx.x; id < npos * IT * nch; id += 256) {
        const int pl_i = id / (IT * nch);
        const int k = (id / nch) % IT;
        const int ch = id % nch;
        const int pg = pT * npos + pl_i;
        const int i = i0 + k;
        if (pg >= p.npix || i >= p.I) continue;
        const uint32_t *wsrc = s_alt + pl_i * plane + (FP4 ? (k * upr) / 2 : k * upr + ch * 4);
        const uint4 val = make_uint4(wsrc[0], wsrc[1], wsrc[2], wsrc[3]);
        const int64_t off = (static_cast<int64_t>(pg) * p.I + i) * p.O2 + o_base;
        uint4 *dst = reinterpret_cast<uint4 *>(p.codes_alt + (FP4 ? off / 2 : off));
        dst[ch] = val;
    }
}

template <bool MAP_A, int BLK, int FMT, int IT, bool DUAL>
__global__ void __launch_bounds__(256, 2) mx_quantize_kernel(const QuantParams p) {
    quantize_tile<MAP_A, BLK, FMT, IT, DUAL>(p, blockIdx.x);
}

// Several tensors of the same format, block mode and code order in one
// launch (e.g. the weights of every layer, quantized together after a weight
// update): CTA b works on tile b - tile0[i] of tensor i, tile0[i] <= b <
// tile0[i + 1].  Small tensors (a 3x3 kernel has 9 spatial positions, so 9
// of a warp's 32 lanes work) then run side by side instead of one after the
// other.
constexpr int kMaxQuantBatch = 16;
struct QuantBatch {
    QuantParams q[kMaxQuantBatch];
    int32_t tile0[kMaxQuantBatch + 1];
    int32_t n;
};

template <bool MAP_A, int BLK, int FMT, bool DUAL>
__global__ void __launch_bounds__(256, 2) mx_quantize_batch_kernel(const __grid_constant__ QuantBatch b) {
    int i = 0;
    while (i + 1 < b.n && static_cast<int>(blockIdx.x) >= b.tile0[i + 1]) ++i;
    quantize_tile<MAP_A, BLK, FMT, 32, DUAL>(b.q[i], static_cast<int>(blockIdx.x) - b.tile0[i]);
}

template <bool MAP_A, int BLK, int FMT>
inline void launch_quantize_batch_fmt(const QuantBatch &b, bool dual, unsigned grid, cudaStream_t s) {
    if (dual) mx_quantize_batch_kernel<MAP_A, BLK, FMT, true><<<grid, 256, 0, s>>>(b);
    else mx_quantize_batch_kernel<MAP_A, BLK, FMT, false><<<grid, 256, 0, s>>>(b);
}

template <bool MAP_A, int BLK>
inline void launch_quantize_batch_blk(const QuantBatch &b, int fmt, bool dual, unsigned grid, cudaStream_t s) {
    if (fmt == 0) launch_quantize_batch_fmt<MAP_A, BLK, 0>(b, dual, grid, s);
    else if (fmt == 1) launch_quantize_batch_fmt<MAP_A, BLK, 1>(b, dual, grid, s);
    else launch_quantize_batch_fmt<MAP_A, BLK, 2>(b, dual, grid, s);
}

template <bool MAP_A>
inline void launch_quantize_batch(const QuantBatch &b, int blk, int fmt, bool dual, unsigned grid, cudaStream_t s) {
    if (blk == kAlongI) launch_quantize_batch_blk<MAP_A, kAlongI>(b, fmt, dual, grid, s);
    else if (blk == kAlongO) launch_quantize_batch_blk<MAP_A, kAlongO>(b, fmt, dual, grid, s);
    else launch_quantize_batch_blk<MAP_A, kSquare>(b, fmt, dual, grid, s);
}

// Host-side dispatch over the compile-time variants.
template <bool MAP_A, int BLK, int FMT, int IT>
inline void launch_quantize_variant(const QuantParams &p, bool dual, unsigned grid, cudaStream_t s) {
    if (dual) mx_quantize_kernel<MAP_A, BLK, FMT, IT, true><<<grid, 256, 0, s>>>(p);
    else mx_quantize_kernel<MAP_A, BLK, FMT, IT, false><<<grid, 256, 0, s>>>(p);
}

template <bool MAP_A, int BLK, int FMT>
inline void launch_quantize_it(const QuantParams &p, bool dual, int it, unsigned grid, cudaStream_t s) {
    if constexpr (FMT != 2) {
        if (it == 16) {
            launch_quantize_variant<MAP_A, BLK, FMT, 16>(p, dual, grid, s);
            return;
        }
    }
    launch_quantize_variant<MAP_A, BLK, FMT, 32>(p, dual, grid, s);
}

template <bool MAP_A, int BLK>
inline void launch_quantize_fmt(const QuantParams &p, bool dual, int it, unsigned grid, cudaStream_t s) {
    if (p.fmt == 0) launch_quantize_it<MAP_A, BLK, 0>(p, dual, it, grid, s);
    else if (p.fmt == 1) launch_quantize_it<MAP_A, BLK, 1>(p, dual, it, grid, s);
    else launch_quantize_it<MAP_A, BLK, 2>(p, dual, it, grid, s);
}

template <bool MAP_A>
inline void launch_quantize_blk(const QuantParams &p, int blk, bool dual, int it, unsigned grid, cudaStream_t s) {
    if (blk == kAlongI) launch_quantize_fmt<MAP_A, kAlongI>(p, dual, it, grid, s);
    else if (blk == kAlongO) launch_quantize_fmt<MAP_A, kAlongO>(p, dual, it, grid, s);
    else launch_quantize_fmt<MAP_A, kSquare>(p, dual, it, grid, s);
}

}  // namespace mqc

namespace mqc {

// ---------------------------------------------------------------------------
// Staged variant for the common case: FP8 codes, the spatial positions of the
// source contiguous (NCHW-like, H*W flattened) and every plane 16-byte
// aligned.  A CTA copies its whole fp32 tile (PT positions x OT rows of the
// primary order's outer axis x IT of its inner axis, 64 KB) into shared
// memory with 16-byte cp.async, all copies in flight at once, then works from
// shared memory only: block maxima (pass 0), the primary rows (pass 1) and
// the second code order (pass 2).  Three CTAs per SM keep about 200 KB of
// loads in flight per SM.  Same arithmetic as mx_quantize_kernel: value times
// the exact power of two 2^-e, then cvt.rn.satfinite.
constexpr int kStagedTileBytes = 65536;

struct StagedParams {
    QuantParams q;
    int32_t PT, OT, IT;          // tile extents (PT * OT * IT * 4 = 64 KB)
    int32_t nPT, nOT, nIT;       // tile counts
    int32_t blk;                 // kAlongI, kAlongO or kSquare
    int32_t map_a;               // the inner axis i is A (order BA)
    // stochastic rounding (order BA only): Philox4x64-10 key (seed, 0),
    // counter (element index / 16, offset, 0, 0); element index
    // ((pix*B + b)*A16 + a) with A16 = A rounded up to 16
    uint64_t seed, offset;
    int32_t a16_blocks;          // A16 / 16
};

// Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC 2011) for the counter (c0, c1, 0, 0) and key (k0, 0):
// ten rounds of two 64x64->128-bit products with the published multipliers,
// the key bumped by the published Weyl increments between rounds.
__device__ __forceinline__ void philox4x64_10(uint64_t c0, uint64_t c1, uint64_t k0, uint64_t (&out)[4]) {
    uint64_t c2 = 0, c3 = 0, k1 = 0;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B97F4A7C15ull;
            k1 += 0xBB67AE8584CAA73Bull;
        }
        const uint64_t h0 = __umul64hi(0xD2E7470EE14C6C93ull, c0), l0 = 0xD2E7470EE14C6C93ull * c0;
        const uint64_t h1 = __umul64hi(0xCA5A826395121157ull, c2), l1 = 0xCA5A826395121157ull * c2;
        const uint64_t n0 = h1 ^ c1 ^ k0, n2 = h0 ^ c3 ^ k1;
        c0 = n0;
        c1 = l1;
        c2 = n2;
        c3 = l0;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

// Stochastic rounding of v (already divided by the block scale) to the
// element format with 16 uniform random bits r (paper, section III-A, Eq. 6:
// gradients are rounded stochastically).  |v| lies between neighbouring
// magnitudes lo <= |v| < hi; with f = (|v| - lo) / (hi - lo) the magnitude
// becomes hi when r < f * 2^16, else lo.  Above the largest finite magnitude
// it saturates; the sign is kept.  In the format's normal range lo is |v|
// with the fp32 mantissa cut to the format's MB bits, and f * 2^16 is the
// cut-off remainder over 2^(7 - MB); below it |v| is a multiple of the
// subnormal step 2^(EMIN - MB) plus f steps.  Returns the code (8 or 4 bits).
template <int FMT>
__device__ __forceinline__ uint32_t sr_code(float v, uint32_t r) {
    constexpr int MB = FMT == 0 ? 3 : (FMT == 1 ? 2 : 1);
    constexpr int BIAS = FMT == 0 ? 7 : (FMT == 1 ? 15 : 1);
    constexpr int EMIN = 1 - BIAS;                                   // exponent of the smallest normal
    constexpr float VMAX = FMT == 0 ? 448.0f : (FMT == 1 ? 57344.0f : 6.0f);
    constexpr uint32_t CMAX = FMT == 0 ? 0x7Eu : (FMT == 1 ? 0x7Bu : 0x7u);
    constexpr float SUB = FMT == 0 ? 512.0f : (FMT == 1 ? 65536.0f : 2.0f);   // 2^(MB - EMIN)
    constexpr int SIGN = FMT == 2 ? 3 : 7;
    const uint32_t bits = __float_as_uint(v);
    const uint32_t ab = bits & 0x7FFFFFFFu;
    const float a = __uint_as_float(ab);
    uint32_t code;
    if (!(a < VMAX)) {
        code = CMAX;
    } else if (static_cast<int>(ab >> 23) - 127 >= EMIN) {
        const uint32_t rem = ab & ((1u << (23 - MB)) - 1u);
        const uint32_t lo = (static_cast<uint32_t>(static_cast<int>(ab >> 23) - 127 + BIAS) << MB) |
                            ((ab >> (23 - MB)) & ((1u << MB) - 1u));
        code = lo + ((r << (7 - MB)) < rem ? 1u : 0u);
    } else {
        const float t = a * SUB;                                     // exact: a power-of-two scaling
        const uint32_t lo = static_cast<uint32_t>(t);
        const float f = t - static_cast<float>(lo);
        code = lo + (static_cast<float>(r) < f * 65536.0f ? 1u : 0u);
    }
    return ((bits >> 31) << SIGN) | code;
}

__device__ __forceinline__ void cp_async_16(void *smem, const void *gmem, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Four codes of v[0..3] (element k of the group in code position k): 32
// bits for FP8, 16 bits (nibbles, low first) for FP4.
template <int FMT>
__device__ __forceinline__ uint32_t pack4(const float (&v)[4]) {
    if (FMT == 2) return cvt_pair<FMT>(v[0], v[1]) | (cvt_pair<FMT>(v[2], v[3]) << 8);
    return cvt_pair<FMT>(v[0], v[1]) | (cvt_pair<FMT>(v[2], v[3]) << 16);
}

// Stores the packed codes of one row of 16 or 32 codes: h[q] holds codes
// 4q..4q+3 as pack4 gives them; `bytes` = 16 or 32 (FP8) or 16 (FP4, 32 codes).
template <int FMT, int NQ>
__device__ __forceinline__ void store_row(uint8_t *dst, const uint32_t (&h)[NQ], int bytes) {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
    if (FMT == 2) {
        d[0] = make_uint4(h[0] | (h[1 % NQ] << 16), h[2 % NQ] | (h[3 % NQ] << 16), h[4 % NQ] | (h[5 % NQ] << 16),
                          h[6 % NQ] | (h[7 % NQ] << 16));
        return;
    }
    d[0] = make_uint4(h[0], h[1 % NQ], h[2 % NQ], h[3 % NQ]);
    if (NQ == 8 && bytes == 32) d[1] = make_uint4(h[4 % NQ], h[5 % NQ], h[6 % NQ], h[7 % NQ]);
}

// OT, IT: tile extents (16 or 32); PT = positions per tile; NS = threads per
// position.  A thread owns o-rows {sub, sub + NS, ...} in the primary pass and
// i-columns {sub, sub + NS, ...} in the second-order pass (64 values each).
//
// SR: stochastic rounding (order BA): pass 1 draws the random bits of its
// rows (one Philox block per 16 codes of a row) and keeps the codes in
// shared memory; pass 2 reorders those codes instead of converting again,
// so both orders hold the same rounding decisions.
template <int FMT, int BLK, int OT, int IT, bool SR>
__global__ void __launch_bounds__(256, SR ? 2 : 3) mx_quantize_staged_kernel(const __grid_constant__ StagedParams sp) {
    constexpr int PT = kStagedTileBytes / (4 * OT * IT);
    constexpr int NS = 256 / PT;
    constexpr int RO = OT / NS, RI = IT / NS;       // owned rows / columns per thread
    extern __shared__ __align__(16) uint8_t smem_q[];
    float *tile = reinterpret_cast<float *>(smem_q);                        // [o][i][pos]
    float *s_inv = reinterpret_cast<float *>(smem_q + kStagedTileBytes);    // [block][pos]
    int *s_amax = reinterpret_cast<int *>(s_inv + 32 * 64);                 // [pos] (square blocks)
    uint8_t *s_codes = reinterpret_cast<uint8_t *>(s_amax + 64);            // SR: [o][i][pos], one code per byte
    const QuantParams &p = sp.q;
    const int tid = threadIdx.x;
    const int pos = tid % PT, sub = tid / PT;

    int t = blockIdx.x;
    const int pT = t % sp.nPT;
    t /= sp.nPT;
    const int oT = t % sp.nOT;
    const int iT = t / sp.nOT;
    const int p0 = pT * PT, o0 = oT * OT, i0 = iT * IT;
    const int64_t so = sp.map_a ? p.sb : p.sa, si = sp.map_a ? p.sa : p.sb;

    // ---- stage the tile: chunk = 4 positions of one (o, i) row
    {
        constexpr int CPR = PT / 4;          // chunks per row
#pragma unroll 4
        for (int c = tid; c < OT * IT * CPR; c += 256) {
            const int row = c / CPR, pc = c % CPR;
            const int o = row / IT, i = row % IT;
            const int pix = p0 + 4 * pc;
            int bytes = 0;
            const float *g = p.src;
            if (o0 + o < p.O && i0 + i < p.I && pix < p.npix) {
                bytes = 4 * min(4, p.npix - pix);
                g = p.src + (o0 + o) * so + (i0 + i) * si + pix;
            }
            cp_async_16(tile + row * PT + 4 * pc, g, bytes);
        }
        if (BLK == kSquare && tid < PT) s_amax[tid] = 0;
        cp_async_wait_all();
        __syncthreads();
    }
    const int pix = p0 + pos;
    const bool pix_ok = pix < p.npix;
    const int nbA = (p.Ap1 + 31) / 32, nbB = (p.Bp1 + 31) / 32;
    const float *tp = tile + pos;

    // ---- pass 0: block maxima and scales
    if (BLK == kSquare) {
        float m = 0.0f;
#pragma unroll
        for (int r = 0; r < RO; ++r)
#pragma unroll
            for (int i = 0; i < IT; ++i) m = fmaxf(m, fabsf(tp[((sub + NS * r) * IT + i) * PT]));
        atomicMax(s_amax + pos, __float_as_int(m));
        __syncthreads();
        if (sub == 0) {
            const uint32_t c = e8m0_code(__int_as_float(s_amax[pos]), p.emax);
            s_inv[pos] = e8m0_inv(c);
            if (pix_ok) {
                const int bT = sp.map_a ? oT : iT, aT = sp.map_a ? iT : oT;
                p.scales[(static_cast<int64_t>(pix) * nbB + bT) * nbA + aT] = static_cast<uint8_t>(c);
            }
        }
    } else if (BLK == kAlongI) {             // one block per (pos, o) row
#pragma unroll
        for (int r = 0; r < RO; ++r) {
            const int o = sub + NS * r;
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < IT; ++i) m = fmaxf(m, fabsf(tp[(o * IT + i) * PT]));
            const uint32_t c = e8m0_code(m, p.emax);
            s_inv[o * PT + pos] = e8m0_inv(c);
            const int og = o0 + o;
            if (pix_ok) {
                if (sp.map_a) {              // A32: row b = o, block iT along a
                    if (og < p.Bp1) p.scales[(static_cast<int64_t>(pix) * p.Bp1 + og) * nbA + iT] = static_cast<uint8_t>(c);
                } else {                     // B32: column a = o, block iT along b
                    if (og < p.Ap1) p.scales[(static_cast<int64_t>(pix) * nbB + iT) * p.Ap1 + og] = static_cast<uint8_t>(c);
                }
            }
        }
    } else {                                 // one block per (pos, i) column
#pragma unroll
        for (int r = 0; r < RI; ++r) {
            const int i = sub + NS * r;
            float m = 0.0f;
#pragma unroll
            for (int o = 0; o < OT; ++o) m = fmaxf(m, fabsf(tp[(o * IT + i) * PT]));
            const uint32_t c = e8m0_code(m, p.emax);
            s_inv[i * PT + pos] = e8m0_inv(c);
            const int ig = i0 + i;
            if (pix_ok) {
                if (sp.map_a) {              // B32: block oT along b, column a = i
                    if (ig < p.Ap1) p.scales[(static_cast<int64_t>(pix) * nbB + oT) * p.Ap1 + ig] = static_cast<uint8_t>(c);
                } else {                     // A32: row b = i, block oT along a
                    if (ig < p.Bp1) p.scales[(static_cast<int64_t>(pix) * p.Bp1 + ig) * nbA + oT] = static_cast<uint8_t>(c);
                }
            }
        }
    }
    __syncthreads();
    // (SR: every thread stays for the barrier before pass 2)
    if (!SR && !pix_ok) return;

    // ---- pass 1: primary rows [pix][o][i0 .. i0 + IT) (clipped to the padded I1)
    if (pix_ok) {
        const bool full_row = IT == 16 || p.I1 - i0 >= 32;
        float inv_i[BLK == kAlongO ? IT : 1];
        if (BLK == kAlongO) {
#pragma unroll
            for (int i = 0; i < (BLK == kAlongO ? IT : 1); ++i) inv_i[i] = s_inv[i * PT + pos];
        }
        const float inv_sq = BLK == kSquare ? s_inv[pos] : 1.0f;
#pragma unroll
        for (int r = 0; r < RO; ++r) {
            const int o = sub + NS * r;
            if (o0 + o >= p.O) break;
            const float inv_row = BLK == kAlongI ? s_inv[o * PT + pos] : inv_sq;
            uint32_t h[IT / 4];
            if constexpr (SR) {
                // random words of this row: Philox blocks (pix*B + b)*A16/16 + i0/16 + k
                uint64_t rw[IT / 4];
                const uint64_t blk0 = (static_cast<uint64_t>(pix) * p.B + (o0 + o)) * sp.a16_blocks + i0 / 16;
#pragma unroll
                for (int k = 0; k < IT / 16; ++k) {
                    uint64_t w4[4];
                    philox4x64_10(blk0 + k, sp.offset, sp.seed, w4);
#pragma unroll
                    for (int j = 0; j < 4; ++j) rw[4 * k + j] = w4[j];
                }
#pragma unroll
                for (int q = 0; q < IT / 4; ++q) {
                    uint32_t c[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int i = 4 * q + k;
                        const float v = tp[(o * IT + i) * PT] * (BLK == kAlongO ? inv_i[i % (BLK == kAlongO ? IT : 1)] : inv_row);
                        const uint32_t r = static_cast<uint32_t>(rw[i >> 2] >> (16 * (i & 3))) & 0xFFFFu;
                        c[k] = sr_code<FMT>(v, r);
                        s_codes[(o * IT + i) * PT + pos] = static_cast<uint8_t>(c[k]);
                    }
                    h[q] = FMT == 2 ? (c[0] | (c[1] << 4) | (c[2] << 8) | (c[3] << 12))
                                    : (c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24));
                }
            } else {
#pragma unroll
            for (int q = 0; q < IT / 4; ++q) {
                float v[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    v[k] = tp[(o * IT + 4 * q + k) * PT] * (BLK == kAlongO ? inv_i[(4 * q + k) % (BLK == kAlongO ? IT : 1)] : inv_row);
                h[q] = pack4<FMT>(v);
            }
            }
            const int64_t off = (static_cast<int64_t>(pix) * p.O + o0 + o) * p.I1 + i0;   // in codes
            store_row<FMT, IT / 4>(p.codes + (FMT == 2 ? off / 2 : off), h, full_row ? IT : 16);
        }
    }
    if (p.codes_alt == nullptr) return;
    if constexpr (SR) {
        // every row of the tile (all positions) has been converted in pass 1
        __syncthreads();
    }
    if (!pix_ok) return;

    // ---- pass 2: second order rows [pix][i][o0 .. o0 + OT) (clipped to the padded O2)
    {
        const bool full_row = OT == 16 || p.O2 - o0 >= 32;
        float inv_o[BLK == kAlongI ? OT : 1];
        if (BLK == kAlongI) {
#pragma unroll
            for (int o = 0; o < (BLK == kAlongI ? OT : 1); ++o) inv_o[o] = s_inv[o * PT + pos];
        }
        const float inv_sq = BLK == kSquare ? s_inv[pos] : 1.0f;
#pragma unroll
        for (int r = 0; r < RI; ++r) {
            const int i = sub + NS * r;
            if (i0 + i >= p.I) break;
            const float inv_col = BLK == kAlongO ? s_inv[i * PT + pos] : inv_sq;
            uint32_t h[OT / 4];
#pragma unroll
            for (int q = 0; q < OT / 4; ++q) {
                if constexpr (SR) {
                    // rows past O were never converted: their codes are +0
                    uint32_t c[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        c[k] = o0 + 4 * q + k < p.O ? s_codes[((4 * q + k) * IT + i) * PT + pos] : 0u;
                    h[q] = FMT == 2 ? (c[0] | (c[1] << 4) | (c[2] << 8) | (c[3] << 12))
                                    : (c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24));
                } else {
                float v[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    v[k] = tp[((4 * q + k) * IT + i) * PT] * (BLK == kAlongI ? inv_o[(4 * q + k) % (BLK == kAlongI ? OT : 1)] : inv_col);
                h[q] = pack4<FMT>(v);
                }
            }
            const int64_t off = (static_cast<int64_t>(pix) * p.I + i0 + i) * p.O2 + o0;   // in codes
            store_row<FMT, OT / 4>(p.codes_alt + (FMT == 2 ? off / 2 : off), h, full_row ? OT : 16);
        }
    }
}

template <int FMT, int BLK, bool SR>
inline void launch_staged_tiles(const StagedParams &sp, unsigned grid, int smem, cudaStream_t s, cudaError_t &attr_err,
                                bool set_attr) {
    auto pick = [&](auto kernel) {
        if (set_attr) {
            cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) attr_err = e;
        }
        kernel<<<grid, 256, smem, s>>>(sp);
    };
    if constexpr (FMT == 2) {            // FP4 rows are 32 codes (16 bytes): IT = 32
        if (sp.OT == 16) pick(mx_quantize_staged_kernel<FMT, BLK, 16, 32, SR>);
        else pick(mx_quantize_staged_kernel<FMT, BLK, 32, 32, SR>);
    } else {
        if (sp.OT == 16 && sp.IT == 16) pick(mx_quantize_staged_kernel<FMT, BLK, 16, 16, SR>);
        else if (sp.OT == 16) pick(mx_quantize_staged_kernel<FMT, BLK, 16, 32, SR>);
        else if (sp.IT == 16) pick(mx_quantize_staged_kernel<FMT, BLK, 32, 16, SR>);
        else pick(mx_quantize_staged_kernel<FMT, BLK, 32, 32, SR>);
    }
}

template <int FMT, bool SR>
inline void launch_staged(const StagedParams &sp, unsigned grid, int smem, cudaStream_t s, cudaError_t &attr_err,
                          bool set_attr) {
    if (sp.blk == kAlongI) launch_staged_tiles<FMT, kAlongI, SR>(sp, grid, smem, s, attr_err, set_attr);
    else if (sp.blk == kAlongO) launch_staged_tiles<FMT, kAlongO, SR>(sp, grid, smem, s, attr_err, set_attr);
    else launch_staged_tiles<FMT, kSquare, SR>(sp, grid, smem, s, attr_err, set_attr);
}

}  // namespace mqc
