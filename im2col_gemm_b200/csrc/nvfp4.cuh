// nvfp4.cuh -- NVFP4 quantization, the format of the MicroQonv paper's own
// experiments (arXiv:2609.28358, section III-A, Eq. 4-6): a per-tensor FP32
// scale T = max|X| / (448 * 6), an E4M3 scale per block of 16 elements
// B = CastE4M3(max|X_i| / (T * 6)), and E2M1 elements Round(x / (B * T)),
// each step one IEEE fp32 operation in the order the equations write them.
// Blocks run along the A-axis (A16), along the B-axis (B16) or are 16 x 16
// squares over (B, A) (SQ16); codes use the channel-batch-first layout of
// the MX quantizer (E2M1, two per byte), scales one E4M3 byte per block.
//
// Two launches: a maximum over the tensor (atomicMax on the float bits of
// non-negative values), then one thread per 16 x 16 tile of a spatial
// position, positions fastest across threads so that the fp32 loads of a
// warp are contiguous in an NCHW source.
#pragma once

#include "common.cuh"

namespace mqc {

enum NvBlock : int { kNvA16 = 0, kNvB16 = 1, kNvSQ16 = 2 };

struct NvParams {
    const float *src;
    int64_t sb, sa;              // element strides of the B and A axes (positions contiguous)
    int32_t B, A, npix;          // real extents
    int32_t Ap, Bp;              // padded extents of the code order (innermost padded to 32)
    int32_t order;               // 0: BA ([pix][b][a], a innermost), 1: AB
    int32_t block;               // NvBlock
    int32_t ntb, nta;            // 16-tiles along B and A (over the padded extents of both orders)
    uint8_t *codes, *codes_alt, *scales;
    int32_t Ap_alt, Bp_alt;      // padded extents of the second order
    float *tscale;               // [0] T (written), [1] max|X| bits (accumulated by the first launch)
};

// Maximum of |x| over the tensor: per-thread maxima of contiguous planes,
// a warp reduction, one atomicMax per warp on the bits of the non-negative
// float (their order as unsigned integers is the order of the values).
__global__ void nv_amax_kernel(const NvParams p) {
    float m = 0.0f;
    const int64_t total = static_cast<int64_t>(p.B) * p.A * p.npix;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t pix = i % p.npix, ba = i / p.npix;
        const int64_t a = ba % p.A, b = ba / p.A;
        m = fmaxf(m, fabsf(__ldg(p.src + b * p.sb + a * p.sa + pix)));
    }
#pragma unroll
    for (int x = 16; x >= 1; x >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, x));
    if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned int *>(p.tscale + 1), __float_as_uint(m));
}

// E4M3 code nearest to q >= 0 (saturating) and its value.
__device__ __forceinline__ uint32_t nv_e4m3(float q, float &val) {
    uint16_t c2;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c2) : "f"(0.0f), "f"(q));
    const uint32_t c = c2 & 0xFFu;
    // value from the fields: subnormal m * 2^-9, normal (1 + m/8) * 2^(e - 7)
    const uint32_t e = c >> 3, m = c & 7u;
    val = e == 0 ? static_cast<float>(m) * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return c;
}

// Two E2M1 codes of x0, x1 at block scale s (Eq. 6), x0 in the low nibble.
__device__ __forceinline__ uint32_t nv_e2m1x2(float x0, float x1, float s) {
    const float v0 = s > 0.0f ? __fdiv_rn(x0, s) : x0 * 0.0f;
    const float v1 = s > 0.0f ? __fdiv_rn(x1, s) : x1 * 0.0f;
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r) : "f"(v1), "f"(v0));
    return r;
}

__global__ void __launch_bounds__(128) nv_quantize_kernel(const NvParams p) {
    const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    const int64_t ntiles = static_cast<int64_t>(p.npix) * p.ntb * p.nta;
    const float amax = __uint_as_float(*reinterpret_cast<const volatile unsigned int *>(p.tscale + 1));
    const float T = __fdiv_rn(amax, 2688.0f);                 // Eq. 4
    const float d = __fmul_rn(T, 6.0f);
    if (t == 0) p.tscale[0] = T;
    if (t >= ntiles) return;
    const int pix = static_cast<int>(t % p.npix);
    const int64_t r = t / p.npix;
    const int at = static_cast<int>(r % p.nta), bt = static_cast<int>(r / p.nta);
    const int b0 = bt * 16, a0 = at * 16;
    auto X = [&](int b, int a) -> float {
        return (b < p.B && a < p.A) ? __ldg(p.src + b * p.sb + a * p.sa + pix) : 0.0f;
    };
    const int nbA = (p.Ap + 15) / 16, nbB = (p.Bp + 15) / 16;   // scale layout of the primary order
    // ---- block maxima and E4M3 scales (Eq. 5)
    float srow[16];                                            // B * T of row (A16), column (B16) or square
    if (p.block == kNvSQ16) {
        float m = 0.0f;
        for (int i = 0; i < 16; ++i)
            for (int j = 0; j < 16; ++j) m = fmaxf(m, fabsf(X(b0 + i, a0 + j)));
        float bs;
        const uint32_t c = nv_e4m3(T > 0.0f ? __fdiv_rn(m, d) : 0.0f, bs);
        if (b0 < p.Bp && a0 < p.Ap) p.scales[(static_cast<int64_t>(pix) * nbB + bt) * nbA + at] = static_cast<uint8_t>(c);
        const float s = __fmul_rn(bs, T);
#pragma unroll
        for (int i = 0; i < 16; ++i) srow[i] = s;
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float m = 0.0f;
            for (int j = 0; j < 16; ++j)
                m = fmaxf(m, fabsf(p.block == kNvA16 ? X(b0 + i, a0 + j) : X(b0 + j, a0 + i)));
            float bs;
            const uint32_t c = nv_e4m3(T > 0.0f ? __fdiv_rn(m, d) : 0.0f, bs);
            srow[i] = __fmul_rn(bs, T);
            if (p.block == kNvA16) {       // row b0 + i, block at
                if (b0 + i < p.Bp && a0 < p.Ap) p.scales[(static_cast<int64_t>(pix) * p.Bp + b0 + i) * nbA + at] = static_cast<uint8_t>(c);
            } else {                        // column a0 + i, block bt
                if (a0 + i < p.Ap && b0 < p.Bp) p.scales[(static_cast<int64_t>(pix) * nbB + bt) * p.Ap + a0 + i] = static_cast<uint8_t>(c);
            }
        }
    }
    // ---- codes (Eq. 6), one per element from its block's B * T; each order
    // packs rows of 16 along its innermost axis (BA: a, AB: b)
    auto code = [&](int i, int j) -> uint32_t {          // element (b0 + i, a0 + j)
        const float sc = p.block == kNvB16 ? srow[j] : srow[i];
        return nv_e2m1x2(X(b0 + i, a0 + j), 0.0f, sc) & 0xFu;
    };
    for (int pass = 0; pass < 2; ++pass) {
        uint8_t *dst = pass == 0 ? p.codes : p.codes_alt;
        if (dst == nullptr) break;
        const int ord = pass == 0 ? p.order : 1 - p.order;
        const int Ai = pass == 0 ? p.Ap : p.Ap_alt, Bi = pass == 0 ? p.Bp : p.Bp_alt;
        const int outer0 = ord == 0 ? b0 : a0, inner0 = ord == 0 ? a0 : b0;
        const int outer_n = ord == 0 ? p.B : p.A;       // the outer axis is not padded
        const int inner_p = ord == 0 ? Ai : Bi;         // the inner axis is (to 32 codes)
        const int outer_p = ord == 0 ? Bi : Ai;
        if (inner0 >= inner_p) continue;
        for (int o = 0; o < 16 && outer0 + o < outer_n; ++o) {
            uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t c = ord == 0 ? code(o, k) : code(k, o);
                if (k < 8) w0 |= c << (4 * k);
                else w1 |= c << (4 * (k - 8));
            }
            const int64_t off = ((static_cast<int64_t>(pix) * outer_p + outer0 + o) * inner_p + inner0) / 2;
            *reinterpret_cast<uint2 *>(dst + off) = make_uint2(w0, w1);
        }
    }
}

}  // namespace mqc
