// subpixel.cuh -- weights of the input gradient as one sub-pixel GEMM.
//
// The input gradient of a convolution with stride (sh, sw) (MicroQonv paper,
// arXiv:2609.28358, section II-C3, Eq. 2) splits by output phase: input pixel
// (sh i + ah, sw j + aw) receives G_Y[i + dh][j + dw] through kernel tap
// r = ah + pad_h - sh dh, s = aw + pad_w - sw dw wherever that tap exists.
// Over all phases the offsets (dh, dw) span a small window (2 x 2 for a 3x3
// kernel with stride 2 and padding 1), so the whole gradient is ONE
// stride-1 correlation of G_Y with a window kernel whose output channels are
// (phase, input channel): Ws[(dh, dw)][(ah, aw, c)][k] = W[k][c][r][s], zero
// where no tap connects the offset to the phase.  A depth-to-space store puts
// column (ah, aw, c) of GEMM row (n, i, j) at (n, c, sh i + ah, sw j + aw).
//
// This kernel builds Ws from the quantized weights: the codes are copied
// byte for byte (their block scales with them), so the GEMM sums exactly the
// products of the per-phase formulation.
#pragma once

#include "common.cuh"

namespace mqc {

struct SubpixGeom {
    int32_t C, Cs;                 // input channels; GEMM columns sh * sw * C
    int32_t R, S, sh, sw, ph, pw;  // kernel, stride, padding
    int32_t dh0, dw0, Rs, Ss;      // window: offsets dh0 .. dh0 + Rs - 1 (and dw)
    int32_t kpw;                   // bytes of one code row of W (padded K)
    int32_t nkb;                   // K-blocks of a row (one scale each)
    int64_t w_tap_pitch;           // scales of W: tap pitch, K-block pitch, row shift
    int32_t w_kb_pitch, w_row_shift;
};

// tap of W feeding window offset t and GEMM column cs, or -1
__device__ __forceinline__ int subpix_tap(const SubpixGeom &g, int t, int cs, int &c) {
    const int phase = cs / g.C;
    c = cs - phase * g.C;
    const int ah = phase / g.sw, aw = phase - (phase / g.sw) * g.sw;
    const int dh = g.dh0 + t / g.Ss, dw = g.dw0 + t % g.Ss;
    const int r = ah + g.ph - g.sh * dh, s = aw + g.pw - g.sw * dw;
    return (r >= 0 && r < g.R && s >= 0 && s < g.S) ? r * g.S + s : -1;
}

// codes: Ws[t][cs][0 .. kpw) from W[tap][c][0 .. kpw) (16 bytes per thread);
// scales: Ws_s[t][kb][cs] (E8M0; 127 = 1.0 where the codes are zero)
__global__ void __launch_bounds__(256) subpix_weights_kernel(const uint8_t *__restrict__ wcodes,
                                                             const uint8_t *__restrict__ wscales, uint8_t *scodes,
                                                             uint8_t *sscales, const SubpixGeom g) {
    const int chunks = g.kpw / 16;
    const int64_t ncode = int64_t(g.Rs) * g.Ss * g.Cs * chunks;
    const int64_t nscale = int64_t(g.Rs) * g.Ss * g.nkb * g.Cs;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < ncode + nscale;
         i += int64_t(gridDim.x) * blockDim.x) {
        if (i < ncode) {
            const int64_t row = i / chunks;
            const int ch = static_cast<int>(i - row * chunks);
            const int t = static_cast<int>(row / g.Cs), cs = static_cast<int>(row - int64_t(t) * g.Cs);
            int c;
            const int tap = subpix_tap(g, t, cs, c);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (tap >= 0) v = reinterpret_cast<const uint4 *>(wcodes + (int64_t(tap) * g.C + c) * g.kpw)[ch];
            reinterpret_cast<uint4 *>(scodes + row * g.kpw)[ch] = v;
        } else {
            const int64_t j = i - ncode;
            const int cs = static_cast<int>(j % g.Cs);
            const int64_t tk = j / g.Cs;
            const int kb = static_cast<int>(tk % g.nkb), t = static_cast<int>(tk / g.nkb);
            int c;
            const int tap = subpix_tap(g, t, cs, c);
            sscales[j] = tap >= 0 ? wscales[tap * g.w_tap_pitch + int64_t(kb) * g.w_kb_pitch + (c >> g.w_row_shift)]
                                  : static_cast<uint8_t>(127);
        }
    }
}

}  // namespace mqc
