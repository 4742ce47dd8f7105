// widen.cuh -- E2M1 codes to E4M3 codes, element for element.
//
// The block-scaled GEMMs run FP4 (E2M1) operands through the same
// kind::mxf8f6f4 tensor-core path as FP8: every E2M1 value (0, 0.5, 1, 1.5,
// 2, 3, 4, 6 and their negatives; OCP MX v1.0 element table) is exactly an
// E4M3 value, so rewriting each 4-bit code as the 8-bit code of the same
// value leaves every product and every E8M0 block scale unchanged (MicroQonv
// paper, arXiv:2609.28358, section III-A: the microscaled product is element
// value x shared scale).  Packed codes hold element 2i in the low nibble of
// byte i; the layout around them (positions, rows, padding) is kept, one byte
// per element instead of half a byte.
#pragma once

#include "common.cuh"

namespace mqc {

// E4M3 code of the E2M1 magnitude code m (0..7): 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ uint32_t e2m1_to_e4m3(uint32_t nib) {
    const uint32_t mag = nib & 7u;
    // 0.5 = 2^-1 -> exponent field 6; 1 and 1.5 -> 7; 2 and 3 -> 8; 4 and 6 -> 9
    const uint32_t code = mag == 0u ? 0u : (mag == 1u ? 0x30u : (((mag >> 1) + 6u) << 3) | ((mag & 1u) << 2));
    return code | ((nib & 8u) << 4);
}

// out[2i] = E4M3(low nibble of in[i]), out[2i + 1] = E4M3(high nibble); 16
// input bytes per thread; nbytes is a multiple of 16 and both buffers are
// 16-byte aligned.
__global__ void __launch_bounds__(256) widen_e2m1_kernel(const uint8_t *__restrict__ in, uint8_t *__restrict__ out,
                                                         int64_t nchunks) {
    for (int64_t c = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; c < nchunks; c += int64_t(gridDim.x) * blockDim.x) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(in) + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t lo = 0u, hi = 0u;
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const uint32_t byte = (w[k] >> (8 * b)) & 0xFFu;
                lo |= (e2m1_to_e4m3(byte & 0xFu) | (e2m1_to_e4m3(byte >> 4) << 8)) << (16 * b);
            }
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const uint32_t byte = (w[k] >> (8 * (b + 2))) & 0xFFu;
                hi |= (e2m1_to_e4m3(byte & 0xFu) | (e2m1_to_e4m3(byte >> 4) << 8)) << (16 * b);
            }
            o[2 * k] = lo;
            o[2 * k + 1] = hi;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out) + 2 * c;
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

}  // namespace mqc
