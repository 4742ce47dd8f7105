// im2col.cuh -- explicit channel-batch-first im2col on quantized codes and
// scales (MicroQonv paper, arXiv:2609.28358, section IV-A): the expansion
// X'_{Cin,N} in (Kh Kw Cin) x (Hout Wout N) form, emitted in the same
// quantized layout as its input (spatial Hout x Wout, B-axis N, A-axis
// (r, s, c) with Ap channels per tap).  Because each spatial position of the
// source holds a contiguous block, every tap of every output position is a
// straight copy of one source chunk (or zeros in the padding): the kernel is
// a 16-byte-vector gather, bound by HBM bandwidth.
#pragma once

#include "common.cuh"

namespace mqc {

struct Im2colParams {
    const uint8_t *src;
    uint8_t *dst;
    int64_t chunk;        // bytes of one contiguous source chunk
    int64_t per_pix;      // source chunks per spatial position (BA: Bp rows; AB: 1 plane)
    int32_t RS, S, P, Q, H, W;
    int32_t st_h, st_w, pad_h, pad_w;
    int64_t n_out;        // total 16-byte units (codes) or bytes (scales) of the output
};

// dst is [pix_out][row][tap][chunk] (row = b for order BA, or the whole
// position plane for order AB with per_pix = 1); src is [pix][row][chunk].
// VEC: copy 16-byte units (codes, chunk a multiple of 16) or single bytes.
template <bool VEC>
__global__ void im2col_gather_kernel(const Im2colParams p) {
    const int64_t unit = VEC ? 16 : 1;
    const int64_t units_per_chunk = p.chunk / unit;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < p.n_out;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        int64_t t = idx;
        const int64_t x = t % units_per_chunk;
        t /= units_per_chunk;
        const int tap = static_cast<int>(t % p.RS);
        t /= p.RS;
        const int64_t row = t % p.per_pix;
        const int64_t pq = t / p.per_pix;
        const int pp = static_cast<int>(pq / p.Q), qq = static_cast<int>(pq % p.Q);
        const int r = tap / p.S, s = tap % p.S;
        const int h = pp * p.st_h + r - p.pad_h, w = qq * p.st_w + s - p.pad_w;
        const bool inside = h >= 0 && h < p.H && w >= 0 && w < p.W;
        const int64_t so = ((static_cast<int64_t>(h) * p.W + w) * p.per_pix + row) * p.chunk + x * unit;
        if (VEC) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (inside) v = __ldg(reinterpret_cast<const uint4 *>(p.src + so));
            reinterpret_cast<uint4 *>(p.dst)[idx] = v;
        } else {
            p.dst[idx] = inside ? __ldg(p.src + so) : static_cast<uint8_t>(0);
        }
    }
}

}  // namespace mqc
