// quantize.cuh -- single-pass OCP-MX quantization into the channel-batch-first
// layout (MicroQonv paper, arXiv:2609.28358: section III-A for the
// microscaling steps with the OCP E8M0 shared scale, section IV-B for the
// quantization directions, section IV-A / Fig. 3 for the layout).
//
// One CTA (8 warps) handles a tile of 32 spatial positions x 32 x 32 of the
// (B, A) plane.  Lane = spatial position, so the fp32 reads along the
// flattened H*W axis of an NCHW source are coalesced.  A thread owns 32
// elements along the primary order's innermost axis ("i") for 4 positions of
// the other axis ("o"); it loads all 128 values, forms the block amax (in
// registers when the block runs along i, with shared-memory atomics when it
// runs along o or is a 32x32 square), converts with cvt.rn.satfinite and
// stores its code rows directly.  The optional second code order goes through
// a shared-memory transpose.
#pragma once

#include "common.cuh"

namespace mqc {

struct QuantParams {
    const float *src;
    int64_t sb, sa, sh, sw;     // element strides of the B, A, H, W axes
    int32_t B, A, H, W;         // real extents
    int32_t npix;               // H * W
    // primary order: codes[(pix*O1 + o)*I1 + i]  (I1 padded innermost extent)
    uint8_t *codes;
    int32_t I1, O1;
    // optional second order: codes_alt[(pix*I + i)*O2 + o] (O2 padded)
    uint8_t *codes_alt;
    int32_t O2;
    uint8_t *scales;
    int32_t Ap1, Bp1;           // primary padded extents, for the scale layout
    int32_t block;              // 0 A32, 1 B32, 2 SQ32
    int32_t fmt;                // 0 E4M3, 1 E5M2, 2 E2M1
    int32_t emax;               // emax_elem of fmt
    int32_t nIT, nOT;           // tile counts along i and o
    int32_t I, O;               // real extents along i and o
};

// E8M0 code of a block whose absolute maximum has fp32 bit pattern `abits`:
// e = floor(log2 amax) - emax, clamped below at -127 (so zero and subnormal
// maxima give 0x00); a non-finite maximum gives 0xFF.
__device__ __forceinline__ uint32_t e8m0_code(uint32_t abits, int emax) {
    if (abits >= 0x7F800000u) return 0xFFu;
    const int ex = static_cast<int>(abits >> 23);
    if (ex == 0) return 0u;
    const int c = ex - emax;
    return c < 0 ? 0u : static_cast<uint32_t>(c);
}

// 2^-e for the scale code (exact power of two, always a normal float).
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

// MAP_A: the thread's 32-element axis i is A (primary order BA); otherwise it
// is B (primary order AB).  FP4: 4-bit codes, two per byte.
template <bool MAP_A, bool FP4>
__global__ void __launch_bounds__(256, 1) mx_quantize_kernel(const QuantParams p) {
    __shared__ uint32_t s_amax[32 * 33];
    // transposed tile for the second order: per position 32 rows of 8 units
    // (4 codes each), plane pitch padded by one word to spread the banks
    __shared__ uint32_t s_alt[32 * 257];

    const int lane = threadIdx.x & 31;
    const int wi = threadIdx.x >> 5;
    int64_t t = blockIdx.x;
    const int pixT = static_cast<int>(t % ((p.npix + 31) / 32));
    t /= (p.npix + 31) / 32;
    const int oT = static_cast<int>(t % p.nOT);
    const int iT = static_cast<int>(t / p.nOT);

    const int pix = pixT * 32 + lane;
    const bool pix_ok = pix < p.npix;
    const int h = pix_ok ? pix / p.W : 0;
    const int w = pix_ok ? pix % p.W : 0;
    const int o0 = oT * 32 + wi * 4;
    const int i0 = iT * 32;

    const bool along_i = (p.block == 0) == MAP_A && p.block != 2;   // A32 & MAP_A, or B32 & !MAP_A
    const bool along_o = (p.block == 1) == MAP_A && p.block != 2;
    const bool sq = p.block == 2;

    if (threadIdx.x < 32 * 33 / 8) {
        for (int k = threadIdx.x; k < 32 * 33; k += 32 * 33 / 8) s_amax[k] = 0u;
    }

    // ---- load 4 x 32 values (zeros outside the real extents)
    float v[4][32];
    const float *base = p.src + static_cast<int64_t>(h) * p.sh + static_cast<int64_t>(w) * p.sw;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = o0 + j;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const int i = i0 + k;
            const int b = MAP_A ? o : i;
            const int a = MAP_A ? i : o;
            v[j][k] = 0.0f;
            if (pix_ok && o < p.O && i < p.I) v[j][k] = __ldcs(base + b * p.sb + a * p.sa);
        }
    }
    __syncthreads();   // s_amax cleared

    // ---- block maxima (integer max of |x| bit patterns orders like |x|)
    uint32_t code_j[4] = {0u, 0u, 0u, 0u};
    if (along_i) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t m = 0u;
#pragma unroll
            for (int k = 0; k < 32; ++k) m = max(m, __float_as_uint(v[j][k]) & 0x7FFFFFFFu);
            code_j[j] = e8m0_code(m, p.emax);
        }
    } else if (along_o) {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            uint32_t m = 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) m = max(m, __float_as_uint(v[j][k]) & 0x7FFFFFFFu);
            atomicMax(&s_amax[k * 33 + lane], m);
        }
    } else {
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int k = 0; k < 32; ++k) m = max(m, __float_as_uint(v[j][k]) & 0x7FFFFFFFu);
        atomicMax(&s_amax[lane], m);
    }
    __syncthreads();

    uint32_t code_sq = 0u;
    if (sq) code_sq = e8m0_code(s_amax[lane], p.emax);

    // ---- scales (layout of the primary order's padded extents)
    const int nbA = (p.Ap1 + 31) / 32, nbB = (p.Bp1 + 31) / 32;
    if (pix_ok) {
        if (along_i) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int o = o0 + j;
                if (MAP_A) {            // A32: row b = o, block iT along a
                    if (o < p.Bp1) p.scales[(static_cast<int64_t>(pix) * p.Bp1 + o) * nbA + iT] = code_j[j];
                } else {                // B32: column a = o, block iT along b
                    if (o < p.Ap1) p.scales[(static_cast<int64_t>(pix) * nbB + iT) * p.Ap1 + o] = code_j[j];
                }
            }
        } else if (along_o) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const int k = wi * 4 + kk;
                const int i = i0 + k;
                const uint32_t c = e8m0_code(s_amax[k * 33 + lane], p.emax);
                if (MAP_A) {            // B32: block oT along b, column a = i
                    if (i < p.Ap1) p.scales[(static_cast<int64_t>(pix) * nbB + oT) * p.Ap1 + i] = c;
                } else {                // A32: row b = i, block oT along a
                    if (i < p.Bp1) p.scales[(static_cast<int64_t>(pix) * p.Bp1 + i) * nbA + oT] = c;
                }
            }
        } else if (wi == 0) {
            const int bT = MAP_A ? oT : iT, aT = MAP_A ? iT : oT;
            p.scales[(static_cast<int64_t>(pix) * nbB + bT) * nbA + aT] = code_sq;
        }
    }

    // ---- convert and store the primary rows; stage the second order
    const int i_bytes = FP4 ? 16 : 32;                        // bytes of one 32-code row
    int row_bytes = (p.I1 - i0) >= 32 ? i_bytes : ((p.I1 - i0) >= 16 ? 16 : 0);
    if (FP4 && p.I1 - i0 < 32) row_bytes = 0;                 // FP4 rows are whole 16-byte units
    uint32_t unit[32];                                         // codes of (k, o0..o0+3) for the alt order
#pragma unroll
    for (int k = 0; k < 32; ++k) unit[k] = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t words[8];
#pragma unroll
        for (int q = 0; q < (FP4 ? 4 : 8); ++q) {
            uint32_t wv = 0u;
#pragma unroll
            for (int e = 0; e < (FP4 ? 8 : 4); e += 2) {
                const int k = q * (FP4 ? 8 : 4) + e;
                float inv0, inv1;
                if (along_i) {
                    inv0 = inv1 = e8m0_inv(code_j[j]);
                } else if (along_o) {
                    inv0 = e8m0_inv(e8m0_code(s_amax[k * 33 + lane], p.emax));
                    inv1 = e8m0_inv(e8m0_code(s_amax[(k + 1) * 33 + lane], p.emax));
                } else {
                    inv0 = inv1 = e8m0_inv(code_sq);
                }
                const float x0 = v[j][k] * inv0, x1 = v[j][k + 1] * inv1;
                uint32_t pair;
                if (FP4) {
                    pair = cvt_e2m1x2(x0, x1);
                    wv |= pair << (4 * e);
                    unit[k] |= (pair & 0xFu) << (4 * j);
                    unit[k + 1] |= (pair >> 4) << (4 * j);
                } else {
                    pair = p.fmt == 1 ? cvt_e5m2x2(x0, x1) : cvt_e4m3x2(x0, x1);
                    wv |= pair << (8 * e);
                    unit[k] |= (pair & 0xFFu) << (8 * j);
                    unit[k + 1] |= (pair >> 8) << (8 * j);
                }
            }
            words[q] = wv;
        }
        const int o = o0 + j;
        if (pix_ok && o < p.O1 && row_bytes > 0) {
            const int64_t off = (static_cast<int64_t>(pix) * p.O1 + o) * p.I1 + i0;
            uint4 *dst = reinterpret_cast<uint4 *>(p.codes + (FP4 ? off / 2 : off));
            dst[0] = make_uint4(words[0], words[1], words[2], words[3]);
            if (!FP4 && row_bytes == 32) dst[1] = make_uint4(words[4], words[5], words[6], words[7]);
        }
    }
    if (p.codes_alt == nullptr) return;

    // units: FP8 -> 32-bit word (4 codes); FP4 -> 16 bits (4 nibbles)
    if (FP4) {
        uint16_t *s16 = reinterpret_cast<uint16_t *>(s_alt);
#pragma unroll
        for (int k = 0; k < 32; ++k) s16[lane * 514 + k * 8 + wi] = static_cast<uint16_t>(unit[k]);
    } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) s_alt[lane * 257 + k * 8 + wi] = unit[k];
    }
    __syncthreads();

    // rows (position, i) of o-codes [oT*32, oT*32+32) clipped to the padded O2
    const int o_base = oT * 32;
    const int alt_bytes_full = FP4 ? 16 : 32;
    int alt_bytes = (p.O2 - o_base) >= 32 ? alt_bytes_full : ((p.O2 - o_base) >= 16 ? 16 : 0);
    if (FP4 && p.O2 - o_base < 32) alt_bytes = 0;
    if (alt_bytes == 0) return;
    const int nch = alt_bytes / 16;
    for (int id = threadIdx.x; id < 32 * 32 * nch; id += 256) {
        const int pl = id / (32 * nch);
        const int k = (id / nch) % 32;
        const int ch = id % nch;
        const int pg = pixT * 32 + pl;
        const int i = i0 + k;
        if (pg >= p.npix || i >= p.I) continue;
        uint4 val;
        if (FP4) {
            const uint32_t *wsrc = s_alt + (pl * 514 + k * 8) / 2;
            val = make_uint4(wsrc[0], wsrc[1], wsrc[2], wsrc[3]);
        } else {
            const uint32_t *wsrc = s_alt + pl * 257 + k * 8 + ch * 4;
            val = make_uint4(wsrc[0], wsrc[1], wsrc[2], wsrc[3]);
        }
        const int64_t off = (static_cast<int64_t>(pg) * p.I + i) * p.O2 + o_base;
        uint4 *dst = reinterpret_cast<uint4 *>(p.codes_alt + (FP4 ? off / 2 : off));
        dst[ch] = val;
    }
}

}  // namespace mqc
