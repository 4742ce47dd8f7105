// conv_gemm.cuh -- block-scaled tcgen05 implicit GEMM for the three
// convolution GEMMs of the MicroQonv paper (arXiv:2609.28358, section II-C3
// and section IV-B):
//     forward        Y_f{Cout,N}   = W_f{Cout,Cin}   . X'_{Cin,N}
//     input grad.    G_X'{Cin,N}   = W_f^T{Cout,Cin} . G_Yf{Cout,N}
//     weight grad.   G_Wf{Cout,Cin} = G_Yf{Cout,N}   . X'^T_{Cin,N}
// with the channel-batch-first im2col (section IV-A) folded into the operand
// staging: the expanded X' is never written.  Each K-block of 32 elements of
// an operand row is one OCP MX block with its own E8M0 scale, and the tensor
// core applies both operands' scales per K-block (Eq. 7: the quantization
// direction matches the dot-product direction).
//
// Two kinds share one kernel:
//   CONV  (forward, input gradient): GEMM rows = output pixels (q, p, n),
//         columns = output channels, reduction = (kernel tap, channel).  The
//         A tile of a tap is one TMA box of the activation tensor at shifted
//         coordinates (out-of-range rows are zero-filled: the padding);
//         strided convolutions use one tensor map per stride phase.
//         The input gradient of a strided convolution can also run as one
//         sub-pixel GEMM: rows = super-pixels, columns = (stride phase,
//         channel), stored depth-to-space (d2s below).
//   WGRAD (weight gradient): rows = C_out, columns = C_in of one tap or
//         (tap, C_in) of a tap group, reduction = (output pixel, batch) with
//         N contiguous; split over K.
//
// CTA layout (persistent, one CTA per SM; 16 warps for CONV, 12 for WGRAD):
//   warp 0      TMA producer (codes of A and B, one elected thread)
//   warp 1      TMEM allocator + MMA issuer (one elected thread): scale
//               factors smem -> TMEM with tcgen05.cp, then tcgen05.mma
//               block_scale, 4 or 8 K-blocks (of 32) per pipeline stage
//   warps 2, 3, 8, 10, 11   scale-factor gather: E8M0 bytes of every operand
//               row and K-block into the 128x4 shared-memory atoms the MMA
//               expects (one stage per warp in turn)
//   warps 4-7   epilogue: TMEM -> registers -> fp32 global stores
//   warps 12-15 (CONV) a second epilogue team, alternate accumulators
// Every wait is bounded in time; a wait that runs out records a device error
// and the CTA winds down without hanging.
#pragma once

#include "common.cuh"

namespace mqc {

constexpr int kMaxTaps = 64;
constexpr int kMaxPhases = 4;   // CONV: output stride phases sharing one launch
constexpr int kGemmThreads = 384;
// Warp roles (a warp's SM sub-partition is its index modulo 4):
//   0 TMA producer, 1 MMA issuer (alone on its sub-partition apart from the
//   epilogue warps), 4-7 epilogue (one per TMEM lane quadrant), and the
//   scale-factor gather warps below; warp 9 only joins the final barrier.
//   CONV kernels have 16 warps: 12-15 are a second epilogue team, the two
//   teams taking alternate accumulators (when there are at least two).
template <int KIND>
__host__ __device__ constexpr int gemm_threads() { return KIND == 0 ? 512 : kGemmThreads; }
constexpr int kNumSfWarps = 5;
__device__ __forceinline__ int sf_warp_index(int warp) {
    return warp == 2 ? 0 : warp == 3 ? 1 : warp == 8 ? 2 : warp == 10 ? 3 : warp == 11 ? 4 : -1;
}
constexpr int kTmemCols = 512;
constexpr int kMaxAcc = 4;       // accumulator ring: tiles between the MMA issuer and the epilogue
constexpr int kSfTmemBase = 256;

enum GemmKind : int { kConv = 0, kWgrad = 1 };

// Where the E8M0 scale of (row, K-block) of an operand lives:
//   base + pixel*pix_pitch + (row >> row_shift)*row_pitch + kblock*kb_pitch (+ tap*tap_pitch)
struct ScaleSrc {
    const uint8_t *base;
    int64_t pix_pitch;
    int64_t tap_pitch;
    int32_t row_shift;     // 5 when 32 rows share a scale (square blocks), else 0
    int32_t row_pitch;
    int32_t kb_pitch;
    int32_t rows;
    int32_t H, W;
    int32_t nblk;          // packed FP4: scale blocks along K per row (bytes past them read as 0);
                           // kb_pitch is then the distance between consecutive blocks
};

struct ConvTap {
    int16_t dh, dw;        // offsets of the A (CONV) or B (WGRAD) tensor-map coordinates
    int16_t sf_dh, sf_dw;  // offsets of the pixel whose scales apply
    int16_t map;           // tensor map (stride phase) of the shifted operand
    int16_t btap;          // CONV: tap index of W; WGRAD: output offset r*S + s
    int16_t aw;            // CONV with interleaved rows: the interleave slot this tap feeds
};

struct alignas(64) GemmParams {
    CUtensorMap amap[4];
    CUtensorMap bmap[4];
    ScaleSrc sfa, sfb;
    ConvTap taps[kMaxTaps];
    int32_t ntaps;
    int32_t n_amaps, n_bmaps;    // tensor maps in use
    int32_t BN, nb_atoms, wkb, stages, nacc, lg_nacc;   // nacc accumulators in TMEM (1, 2 or 4)
    int32_t kbs;                 // K-blocks (of 32) per pipeline stage: 4 or 8
    uint32_t idesc;
    uint64_t timeout_ns;
    int32_t num_units;
    int32_t a_box_bytes, b_box_bytes;
    // rows between consecutive K sub-tiles (of wkb K-blocks) inside a group
    // of 4 K-blocks in shared memory: 128 / BN when each sub-tile is its own
    // box (CONV), the box rows when one box spans the group (WGRAD, whose
    // boxes hold only the rows that exist)
    int32_t a_slab, b_slab;
    // CONV kind
    int32_t rows_nfirst;         // A map dims (C, N, W, H) instead of (C, W, H, N)
    // rows interleaved along the output width: tile row m = aw + sub * (q +
    // bq * (p + bp * n)) lands on output column sub * q + aw.  The input
    // gradient of a stride-s convolution uses sub = s: a tap feeds only the
    // rows of its slot aw, the other rows of its A box are zero (the box
    // reads them out of range).  sub = 1 otherwise.
    int32_t sub;
    int32_t sf_vec4;             // A: each group of 4 K-blocks is 4 aligned consecutive scale bytes (one tap)
    int32_t sfb_vec4;            // B: likewise (the weights' scales along C)
    int32_t sfb_cached;          // CONV: B scale atoms of every (column tile, group) built once per CTA
    int32_t sq_gather;           // WGRAD: square blocks on both operands, 16-row groups of an atom aligned
    int32_t sq16;                // WGRAD, sq_gather: a 32-row group of B may hold two taps (cpad = 16 mod 32)
    int32_t groups;              // CONV: groups of 4 K-blocks per tile
    // scale-gather warps in use (at most 5 and at most the stages; 0: that
    // maximum).  Warp w takes the stages w, w + nsf, ...: with every unit
    // having the same stages, the host picks nsf so that no warp keeps
    // drawing the largest stage of each unit
    int32_t nsf;
    // CONV: a unit is um consecutive 128-row tiles (sub-tiles) sharing the
    // B operand, the pipeline stages and the per-unit bookkeeping; each
    // sub-tile has its own accumulator (um x BN TMEM columns per unit)
    int32_t um, MTILES;
    int32_t bq, bp, bn;          // A box extents along q, p, n
    int32_t TQ, TP, TN, NT;      // tile counts
    int32_t Ne;                  // output extent along n (row mask)
    int32_t CB, total_kb;        // K-blocks per tap, most K-blocks of a tile over the phases
    // CONV output phases (the input gradient of a strided convolution splits
    // its output into stride phases with different tap sets; the forward has
    // one phase).  Units run phase-fastest within a tile so the phases that
    // interleave in memory are written at about the same time.
    int32_t nph;
    int32_t ph_tap0[kMaxPhases];  // first tap of the phase in taps[]
    int32_t ph_tkb[kMaxPhases];   // K-blocks of a tile of the phase
    int32_t ph_gofs[kMaxPhases];  // first group of 4 K-blocks of the phase (scale cache index)
    int32_t ph_Qe[kMaxPhases], ph_Pe[kMaxPhases];   // output extents of the phase (row masks)
    int64_t ph_out_base[kMaxPhases];
    int32_t a_st_h, a_st_w;      // output coordinate -> scale pixel multiplier
    int32_t Ncols;               // GEMM columns (output channels)
    // WGRAD kind: K is walked in "kits" of 4 K-blocks (one TMA box per operand)
    int32_t MT, Mrows, splits, kiters_total, QG, NC, bqk, P, Q;
    // WGRAD tap groups: the GEMM columns of a unit are (tap of the group,
    // input channel), cpad rows per tap (a multiple of 8), so one MMA per
    // K-block covers ntg taps.  ntg = 1: the columns are channels of one tap.
    int32_t ntg, ngroups, cpad;
    // WGRAD window boxes (tap groups of whole kernel rows): bmap[0] covers the
    // unphased X as (batch, C, W, H), and one box of (batch, cpad, S, ntg / S)
    // at the pixel's window origin lands every (tap, channel) row of the
    // group in the column order of the GEMM; wb_S = S, wb_ph/wb_pw = padding
    int32_t wbox, wb_S, wb_ph, wb_pw;
    // WGRAD k16 (batch of at most 16): every operand row holds 16 batch codes
    // in HBM, so a K-block row is 16 bytes in shared memory (the MMA reads its
    // other 16 from a zero block) and the TMA views take 16 rows of 16 bytes
    // as one 256-byte row: (256, rows / 16, ...) boxes, row coordinates / 16
    int32_t k16;
    // CONV k16 (narrow forward: 16-byte code rows and a batch of 16): a
    // pixel's codes of the whole batch are one 256-byte run, the A maps are
    // (256, W', H') and a box of 8 runs is a tile (rows n fastest, bn = 16,
    // bq = 8 or bq x bp = 8 with a quantized output); the MMA reads the upper
    // 16 bytes of every K-block row from the zero block, as for WGRAD
    // sf_pix: square X blocks, so one scale byte per pixel serves all 16
    // rows of the pixel (8 bytes per tap and tile, shared by shuffles)
    // ep_stage: the fp32 tile goes through shared memory as [n][column][q]
    // so that each (n, channel) gets its 8 consecutive q as 16-byte stores
    int32_t sf_pix, ep_stage;
    // CONV ep_vec: the 4 rows of each lane quad are 4 consecutive q of one
    // (p, n) and every output row start is 16-byte aligned: the epilogue
    // transposes 4 x 4 blocks across the quad and stores 16-byte runs (in the
    // instances with the 32-bit scale gather or units of several tiles only:
    // in the others the extra code measured slower on the sub-pixel input
    // gradient and gained nothing)
    int32_t ep_vec;
    // CONV d2s (input gradient as one sub-pixel GEMM): GEMM column n is
    // (phase n / cpad, channel n % cpad) and lands at channel offset
    // (n % cpad) * os_c + d2s_off[phase]; cpad is a multiple of 16.
    // d2s = 2: width stride 2 and column tiles of whole phase pairs
    // (aw = 0, 1): the two are stored together, 8 bytes per lane
    int32_t d2s;
    int64_t d2s_off[kMaxPhases];
    // the divisions of the unit and row decoding, by launch constants
    FastDiv fd_NT, fd_nph, fd_TQ, fd_TP, fd_sub, fd_bq, fd_bp, fd_bn, fd_MT, fd_ngroups, fd_splits, fd_cpad;
    int32_t x_st_h, x_st_w;      // stride of X pixels per output pixel
    // CONV QOUT (forward with a quantized output, template flag): the
    // epilogue applies the activation and writes the result as the next
    // layer's MX-quantized input [N][K][P][Q] (B-axis N, A-axis K): codes in
    // order BA [P][Q][N][q_Kp], optionally order AB [P][Q][K][q_Np], one
    // E8M0 scale per block of 32 channels (A32) or per 32 x 32 square over
    // (n, k) (SQ32); rows run n fastest within a pixel (rows_nfirst) with bn =
    // q_lanes (16 or 32), so a square's rows are lanes of one warp
    uint8_t *q_codes, *q_codes_alt, *q_scales;
    float *q_y;                  // optional fp32 copy of the activated output (NCHW), else null
    int32_t q_fmt, q_sq, q_act, q_emax, q_Kp, q_Np, q_nbA, q_nbB, q_lanes;
    // CONV PK (template parameter, packed FP4 operands: the E2M1 codes as
    // stored, a 32-byte K-block holds 64 elements):
    //   PK = 1  OCP MXFP4, two E8M0 scales per row and K-block (blocks of 32
    //           along C), two K-blocks per scale atom, kind::mxf4 scale_vec::2X
    //   PK = 2  NVFP4, four UE4M3 scales per row and K-block (blocks of 16),
    //           one atom per K-block, kind::mxf4nvf4 scale_vec::4X; the
    //           epilogue multiplies by the per-tensor scales nv_tx[0] * nv_tw[0]
    const float *nv_tx, *nv_tw;
    int32_t pk;
    // output
    float *out;
    int64_t out_base, os_q, os_p, os_n, os_c, os_m, split_pitch;
};

struct UnitInfo {
    int nk;                 // pipeline stages of this unit
    int nt;                 // column tile
    int mt0;                // CONV: first 128-row tile of the unit
    int ph, tap0, tkb;      // CONV: output phase, its first tap and K-blocks
    int kbase, nkit;        // WGRAD: first kit and number of kits
    int q0, p0, n0;         // CONV: tile origin
    int m0;                 // WGRAD: first output channel row
    int col0;               // first GEMM column
    int tap, tig;           // WGRAD: first tap of the unit's group, taps in the group
    int split;              // WGRAD: split index
};

template <int KIND>
__device__ __forceinline__ UnitInfo decode_unit(const GemmParams &p, int u) {
    UnitInfo I{};
    if (KIND == kConv) {
        const uint32_t r = p.fd_NT.div(u);
        const int nt = u - static_cast<int>(r) * p.NT;
        const uint32_t mg = p.fd_nph.div(r);
        const int ph = static_cast<int>(r - mg * p.nph);
        const uint32_t mt = mg * p.um;
        I.mt0 = static_cast<int>(mt);
        const uint32_t m2 = p.fd_TQ.div(mt);
        const int tq = static_cast<int>(mt - m2 * p.TQ);
        const uint32_t tn = p.fd_TP.div(m2);
        const int tp = static_cast<int>(m2 - tn * p.TP);
        I.nt = nt;
        I.q0 = tq * p.bq;
        I.p0 = tp * p.bp;
        I.n0 = static_cast<int>(tn) * p.bn;
        I.col0 = nt * p.BN;
        I.ph = ph;
        I.tap0 = p.ph_tap0[ph];
        I.tkb = p.ph_tkb[ph];
        I.nk = (I.tkb + p.kbs - 1) / p.kbs;
    } else {
        const uint32_t r1 = p.fd_MT.div(u);
        const int mt = u - static_cast<int>(r1) * p.MT;
        const uint32_t r2 = p.fd_NT.div(r1);
        const int nt = static_cast<int>(r1 - r2 * p.NT);
        const uint32_t sp = p.fd_ngroups.div(r2);
        I.tap = static_cast<int>(r2 - sp * p.ngroups) * p.ntg;
        I.tig = min(p.ntg, p.ntaps - I.tap);
        I.split = static_cast<int>(sp);
        I.nt = nt;
        I.m0 = mt * 128;
        I.col0 = nt * p.BN;
        // split s covers kits [s*K/splits, (s+1)*K/splits); s*K < 2^31 (host check)
        const int k0 = static_cast<int>(p.fd_splits.div(static_cast<uint32_t>(I.split * p.kiters_total)));
        const int k1 = static_cast<int>(p.fd_splits.div(static_cast<uint32_t>((I.split + 1) * p.kiters_total)));
        I.kbase = k0;
        I.nkit = k1 - k0;
        const int ga = p.kbs / 4;
        I.nk = (I.nkit + ga - 1) / ga;
    }
    return I;
}

// 4 x 4 transpose across the lanes of a quad: lane e of the quad holds row e
// (x0..x3 = columns 0..3) on entry and column e (x0..x3 = rows 0..3) on exit.
// Two exchange steps, each swapping the off-diagonal halves of 2 x 2 blocks
// (of single entries with lane e ^ 1, then of 2 x 2 blocks with lane e ^ 2).
__device__ __forceinline__ void quad_transpose(uint32_t &x0, uint32_t &x1, uint32_t &x2, uint32_t &x3, int e) {
    const bool odd = (e & 1) != 0, hi = (e & 2) != 0;
    uint32_t a = odd ? x0 : x1, b = odd ? x2 : x3;
    a = __shfl_xor_sync(0xFFFFFFFFu, a, 1);
    b = __shfl_xor_sync(0xFFFFFFFFu, b, 1);
    if (odd) {
        x0 = a;
        x2 = b;
    } else {
        x1 = a;
        x3 = b;
    }
    a = hi ? x0 : x2;
    b = hi ? x1 : x3;
    a = __shfl_xor_sync(0xFFFFFFFFu, a, 2);
    b = __shfl_xor_sync(0xFFFFFFFFu, b, 2);
    if (hi) {
        x0 = a;
        x1 = b;
    } else {
        x2 = a;
        x3 = b;
    }
}

// Row m (0..127) of a CONV tile -> interleave slot and output coordinates
// within the tile.
__device__ __forceinline__ void conv_row(const GemmParams &p, int m, int &aw, int &iq, int &ip, int &in) {
    if (p.rows_nfirst) {
        const uint32_t t = p.fd_bn.div(m);
        in = m - static_cast<int>(t) * p.bn;
        const uint32_t t2 = p.fd_bq.div(t);
        iq = static_cast<int>(t - t2 * p.bq);
        ip = static_cast<int>(t2);
        aw = 0;
    } else {
        const uint32_t t = p.fd_sub.div(m);
        aw = m - static_cast<int>(t) * p.sub;
        const uint32_t t2 = p.fd_bq.div(t);
        iq = static_cast<int>(t - t2 * p.bq);
        const uint32_t t3 = p.fd_bp.div(t2);
        ip = static_cast<int>(t2 - t3 * p.bp);
        in = static_cast<int>(t3);
    }
}

// conv_row of row m packed into one word, decoded once per kernel: the slot
// and the (q, p, n) offsets in bytes 0-3 (each below 128, the slot below
// 256), bit 31 set when m is past the tile's rows.
__device__ __forceinline__ uint32_t conv_row_packed(const GemmParams &p, int m) {
    int aw, iq, ip, in;
    conv_row(p, m, aw, iq, ip, in);
    const bool past = m >= p.sub * p.bq * p.bp * p.bn;
    return static_cast<uint32_t>(aw) | (static_cast<uint32_t>(iq) << 8) | (static_cast<uint32_t>(ip) << 16) |
           (static_cast<uint32_t>(in) << 24) | (past ? 0x80000000u : 0u);
}

// Origin (q, p, n) of the 128-row tile mt of a CONV launch (tiles run q
// fastest, then p, then n; mt past the last tile gives n >= N: all rows out
// of range, its boxes read zeros).
__device__ __forceinline__ void tile_origin(const GemmParams &p, int mt, int &q0, int &p0, int &n0) {
    const uint32_t m2 = p.fd_TQ.div(mt);
    const uint32_t tn = p.fd_TP.div(m2);
    q0 = (mt - static_cast<int>(m2) * p.TQ) * p.bq;
    p0 = (static_cast<int>(m2) - static_cast<int>(tn) * p.TP) * p.bp;
    n0 = static_cast<int>(tn) * p.bn;
}

__device__ __forceinline__ uint32_t swizzle_of(int wkb) {
    return wkb == 4 ? kSwizzle128B : (wkb == 2 ? kSwizzle64B : kSwizzle32B);
}

// Walks K-blocks g = 0, 1, 2, ... of a CONV tile as (tap, channel block)
// without divisions.
struct KbWalker {
    int tap, cb;
    __device__ __forceinline__ void advance(int n, int CB) {
        cb += n;
        while (cb >= CB) {
            cb -= CB;
            ++tap;
        }
    }
};

// Walks the kits of a WGRAD unit as (output row pp, q-group qg, n-chunk nc).
struct KitWalker {
    int nc, qg, pp;
    __device__ __forceinline__ void init(const GemmParams &p, int kit) {
        nc = kit % p.NC;
        qg = (kit / p.NC) % p.QG;
        pp = kit / (p.NC * p.QG);
    }
    __device__ __forceinline__ void next(const GemmParams &p) {
        if (++nc == p.NC) {
            nc = 0;
            if (++qg == p.QG) {
                qg = 0;
                ++pp;
            }
        }
    }
};

// SFV4, CONV: the A scales of 4 consecutive K-blocks are 4 aligned bytes of
// one tap and are read with one 32-bit load per row; otherwise one byte per
// (row, K-block).  SFV4, WGRAD: both operands have 32x32 square blocks, so
// every 32-row group of an A atom and every 16-row group of a B atom (16 | cpad:
// a group stays inside one tap and one channel block) shares one scale per
// K-block; a group of 4 K-blocks needs 4 x 4 A bytes and 2 x 8 x 4 B bytes,
// loaded one or two per lane and merged by warp shuffles (instead of one load
// per row group and K-block in every lane).
// The choice is a template parameter so that each kernel carries only one
// gather path (the per-stage code of all roles has to share the instruction
// cache).
//
// UMT (CONV only): 128-row sub-tiles per unit (1, 2 or 4; p.um equals it).
// A template parameter as well, so that the one-tile kernel carries no
// sub-tile loops.
// Activations the quantized forward output can apply before quantizing:
// 0 none, 1 ReLU, 2 SiLU x / (1 + e^-x), with CUDA's fast exponential and
// division intrinsics (a few ulp; the codes are decided on this fp32 value).
__device__ __forceinline__ float activate(float x, int act) {
    if (act == 1) return fmaxf(x, 0.0f);
    if (act == 2) return __fdividef(x, 1.0f + __expf(-x));
    return x;
}

// E8M0 code of a block maximum and its inverse scale, for the quantized
// forward output: e = floor(log2 amax) - emax, clamped below at -127 (zero
// and subnormal maxima give 0x00); the same rule as the quantizer's.
__device__ __forceinline__ uint32_t qout_scale_code(float amax, int emax) {
    const uint32_t bits = __float_as_uint(amax);
    if (bits >= 0x7F800000u) return 0xFFu;
    const int ex = static_cast<int>(bits >> 23);
    const int c = ex - emax;
    return (ex == 0 || c < 0) ? 0u : static_cast<uint32_t>(c);
}
__device__ __forceinline__ float qout_inv_scale(uint32_t code) {
    if (code == 0xFFu) return __uint_as_float(0x00400000u);
    return __uint_as_float((254u - code) << 23);
}

// Four codes, one per byte (FP4: a nibble in each byte), round-to-nearest-
// even with saturation.
__device__ __forceinline__ uint32_t qout_cvt4(int fmt, float a, float b, float c, float d) {
    uint16_t lo, hi;
    if (fmt == 0) {
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
        return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    if (fmt == 1) {
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
        return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    uint32_t p0, p1;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(p0) : "f"(b), "f"(a));
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(p1) : "f"(d), "f"(c));
    return (p0 & 0xFu) | ((p0 >> 4) << 8) | ((p1 & 0xFu) << 16) | ((p1 >> 4) << 24);
}

// Packs the bytes of w[0..7] (32 codes, one per byte) into 16 bytes of
// nibbles, element 2i in the low nibble.
__device__ __forceinline__ uint4 qout_pack_fp4(const uint32_t (&w)[8]) {
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t a = w[2 * q], b = w[2 * q + 1];
        o[q] = (a & 0xFu) | ((a >> 4) & 0xF0u) | ((a >> 8) & 0xF00u) | ((a >> 12) & 0xF000u) |
               ((b & 0xFu) << 16) | (((b >> 8) & 0xFu) << 20) | (((b >> 16) & 0xFu) << 24) | (((b >> 24) & 0xFu) << 28);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// QOUT: the output tile of one epilogue warp, 32 rows x 32 columns
// (columns k0 .. k0 + 31 of its TMEM lane quadrant) -> activation, block
// maxima, scales, codes in order BA, and through a per-warp 32 x 36-byte
// shared-memory transpose the codes in order AB.
//   v        the 32 accumulator columns of this thread's row
//   row_ok   the row is an output (n < N, pixel inside the output)
//   pix, n   next-layer pixel p*Q + q and batch index of the row
//   k0       first output channel of the 32
//   s_tr     this warp's transposition scratch (32 x 36 bytes)
__device__ __forceinline__ void qout_chunk(const GemmParams &p, const uint32_t (&r)[32], bool row_ok, int pix,
                                           int n, int k0, uint32_t *s_tr, int lane) {
    const int K = p.Ncols;
    float v[32];
    float m = 0.0f;
    if (row_ok && k0 + 32 <= K) {
        // whole chunk inside the output: no per-element masks
        if (p.q_act == 2) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = activate(__uint_as_float(r[j]), 2);
        } else if (p.q_act == 1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = fmaxf(__uint_as_float(r[j]), 0.0f);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = (row_ok && k0 + j < K) ? activate(__uint_as_float(r[j]), p.q_act) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
    if (p.q_y != nullptr && row_ok) {
        // optional fp32 copy, NCHW [N][K][P][Q]: p.os_* give the strides
        float *op = p.q_y + static_cast<int64_t>(n) * p.os_n + static_cast<int64_t>(pix) + static_cast<int64_t>(k0) * p.os_c;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (k0 + j < K) op[j * p.os_c] = v[j];
    }
    if (p.q_sq) {
        // square block: the rows of one pixel are q_lanes consecutive lanes
#pragma unroll
        for (int x = 1; x < 32; x <<= 1)
            if (x < p.q_lanes) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, x));
    }
    const uint32_t code = qout_scale_code(m, p.q_emax);
    const float inv = qout_inv_scale(code);
    // pixel validity of the square's first lane (all rows of a pixel share it)
    if (p.q_sq) {
        const int lead = lane & ~(p.q_lanes - 1);
        const bool pix_ok = __shfl_sync(0xFFFFFFFFu, row_ok ? 1 : 0, lead) != 0;
        if (lane == lead && pix_ok)
            p.q_scales[(static_cast<int64_t>(pix) * p.q_nbB + (n >> 5)) * p.q_nbA + (k0 >> 5)] = static_cast<uint8_t>(code);
    } else if (row_ok) {
        p.q_scales[(static_cast<int64_t>(pix) * p.Ne + n) * p.q_nbA + (k0 >> 5)] = static_cast<uint8_t>(code);
    }
    uint32_t w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) w[q] = qout_cvt4(p.q_fmt, v[4 * q] * inv, v[4 * q + 1] * inv, v[4 * q + 2] * inv, v[4 * q + 3] * inv);
    const bool fp4 = p.q_fmt == 2;
    // order BA: row (pix, n), channels k0 .. k0 + 31 (clipped to the padded q_Kp)
    if (row_ok) {
        const int64_t off = (static_cast<int64_t>(pix) * p.Ne + n) * p.q_Kp + k0;   // in codes
        if (fp4) {
            *reinterpret_cast<uint4 *>(p.q_codes + off / 2) = qout_pack_fp4(w);
        } else {
            uint4 *d = reinterpret_cast<uint4 *>(p.q_codes + off);
            d[0] = make_uint4(w[0], w[1], w[2], w[3]);
            if (p.q_Kp - k0 >= 32) d[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
    if (p.q_codes_alt == nullptr) return;
    // order AB: lane L takes channel k0 + L and the codes of the 32 rows
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 8; ++q) s_tr[lane * 9 + q] = w[q];
    __syncwarp();
    // lane L: byte L % 4 of word L / 4 of every row, four rows per output word
    uint32_t t[8];
    const uint32_t sel = static_cast<uint32_t>(lane & 3) | (static_cast<uint32_t>(4 + (lane & 3)) << 4);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t *col = s_tr + (lane >> 2);
        const uint32_t lo = __byte_perm(col[(4 * q) * 9], col[(4 * q + 1) * 9], sel);
        const uint32_t hi = __byte_perm(col[(4 * q + 2) * 9], col[(4 * q + 3) * 9], sel);
        t[q] = __byte_perm(lo, hi, 0x5410u);
    }
    // pixels and row validity of the lanes' groups
    const int pix0 = __shfl_sync(0xFFFFFFFFu, pix, 0), pix1 = __shfl_sync(0xFFFFFFFFu, pix, 16);
    const int n0 = __shfl_sync(0xFFFFFFFFu, n, 0), n1 = __shfl_sync(0xFFFFFFFFu, n, 16);
    const bool ok0 = __shfl_sync(0xFFFFFFFFu, row_ok ? 1 : 0, 0) != 0;
    const bool ok1 = __shfl_sync(0xFFFFFFFFu, row_ok ? 1 : 0, 16) != 0;
    const int k = k0 + lane;
    if (k >= K) return;
    if (p.q_lanes == 32) {
        // one pixel, batch n0 .. n0 + 31 (clipped to the padded q_Np)
        if (!ok0) return;
        const int64_t off = (static_cast<int64_t>(pix0) * K + k) * p.q_Np + n0;
        if (fp4) {
            *reinterpret_cast<uint4 *>(p.q_codes_alt + off / 2) = qout_pack_fp4(t);
        } else {
            uint4 *d = reinterpret_cast<uint4 *>(p.q_codes_alt + off);
            d[0] = make_uint4(t[0], t[1], t[2], t[3]);
            if (p.q_Np - n0 >= 32) d[1] = make_uint4(t[4], t[5], t[6], t[7]);
        }
    } else {
        // two pixels of 16 rows each (a batch of at most 16: q_Np = 16 FP8 or
        // 32 FP4 codes, the rows past N are zero codes)
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            if (!(g == 0 ? ok0 : ok1)) continue;
            const int64_t off = (static_cast<int64_t>(g == 0 ? pix0 : pix1) * K + k) * p.q_Np;
            if (fp4) {
                uint32_t h[8] = {t[4 * g], t[4 * g + 1], t[4 * g + 2], t[4 * g + 3], 0u, 0u, 0u, 0u};
                *reinterpret_cast<uint4 *>(p.q_codes_alt + off / 2) = qout_pack_fp4(h);
            } else {
                *reinterpret_cast<uint4 *>(p.q_codes_alt + off) = make_uint4(t[4 * g], t[4 * g + 1], t[4 * g + 2], t[4 * g + 3]);
            }
        }
        (void)n1;
    }
}

template <int KIND, bool SFV4, int UMT, bool QOUT = false, int PK = 0, bool NAR = false>
__global__ void __launch_bounds__(gemm_threads<KIND>(), 1) conv_gemm_kernel(const __grid_constant__ GemmParams p) {
    // NAR: the narrow forward (k16 CONV: whole-batch pixel runs, per-pixel
    // scale gather, staged epilogue); its code is only in these instances
    // ROWDEC: the tile rows of the gather and epilogue lanes decoded once per
    // kernel (in the one-tile byte-gather instance the longer-lived registers
    // measured slower on the sub-pixel input gradient, so it decodes per tile)
    constexpr bool ROWDEC = KIND == kConv && (SFV4 || UMT > 1);
    constexpr int SPK = PK == 2 ? 4 : (PK == 1 ? 2 : 1);   // scale bytes per row and K-block = atoms per group
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // swizzled operand tiles need 1024-byte alignment
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int S = p.stages;                   // at least 2
    const int KS = p.kbs;                     // K-blocks per stage
    const int GA = KS / 4;                    // groups of 4 K-blocks (one scale atom) per stage
    const int row_bytes = 32 * p.wkb;         // bytes of one operand row of a TMA box
    const int kb_bytes = p.k16 ? 16 : 32;     // shared-memory bytes of one row of one K-block
    const int srow = p.k16 ? 16 : row_bytes;  // shared-memory bytes of one row of a TMA box (wkb K-blocks)
    const int rsh = p.k16 ? 4 : 0;            // row coordinate shift of the 16-row TMA views
    const int lg_wkb = p.wkb == 4 ? 2 : (p.wkb == 2 ? 1 : 0);
    constexpr int UM = KIND == kConv ? UMT : 1;   // 128-row sub-tiles per unit
    const int a_sub_stage = 128 * kb_bytes * KS;   // one sub-tile's A rows of a stage
    const int a_stage = UM * a_sub_stage;
    const int b_stage = p.BN * kb_bytes * KS;
    const int sfa_stage = 512 * GA * UM * SPK;       // A atoms [group][sub-tile] (NV: [K-block])
    const int sfb_stage = 512 * GA * p.nb_atoms * SPK;
    uint8_t *sA = smem;
    uint8_t *sB = sA + S * a_stage;
    uint8_t *sSFA = sB + S * b_stage;
    uint8_t *sSFB = sSFA + S * sfa_stage;
    uint8_t *sSFBc = sSFB + S * sfb_stage;    // cached B atoms: [column tile][group][atom] x 512 B
    const int sfbc_bytes = p.sfb_cached ? p.NT * p.groups * p.nb_atoms * 512 : 0;
    // full[s]: completes when the TMA bytes of stage s have landed AND the
    // scale-gather warp of stage s has arrived (count 2)
    uint64_t *full = reinterpret_cast<uint64_t *>(sSFBc + sfbc_bytes);
    uint64_t *empty = full + S;
    uint64_t *acc_full = empty + S;
    uint64_t *acc_empty = acc_full + kMaxAcc;
    uint64_t *ep_bar = acc_empty + kMaxAcc;       // ep_stage: one per epilogue team (4 warps)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(ep_bar + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    // k16: the upper 16 bytes of every operand row (batch 16..31 of a K-block)
    // are read by the MMA from this zero block (256 rows x 16 bytes)
    uint8_t *sZ = reinterpret_cast<uint8_t *>(full) + 1024;
    // QOUT: eight 32 x 36-byte transposition buffers (one per epilogue warp);
    // ep_stage: two buffers per team of 16 planes (n) x 260 floats ([column][q]
    // padded by 4, so that the 16 rows n of a store hit 8 banks pairwise)
    uint32_t *sTr = reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(full) + 1024 + (p.k16 ? 4096 : 0));
    float *sEp = reinterpret_cast<float *>(sTr);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 2);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < kMaxAcc; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(&ep_bar[0], 4);
        mbar_init(&ep_bar[1], 4);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < p.n_amaps; ++i) prefetch_tensormap(&p.amap[i]);
        for (int i = 0; i < p.n_bmaps; ++i) prefetch_tensormap(&p.bmap[i]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    if (KIND == kConv && p.sfb_cached) {
        // every thread helps build the B scale atoms once: item = (column tile,
        // group of 4 K-blocks, atom); lane l writes rows l, l+32, l+64, l+96
        const int items = p.NT * p.groups * p.nb_atoms;
        for (int item = warp; item < items; item += gemm_threads<KIND>() / 32) {
            const int at = item % p.nb_atoms;
            const int gq = (item / p.nb_atoms) % p.groups;
            const int nt = item / (p.nb_atoms * p.groups);
            int ph = 0;
            while (ph + 1 < p.nph && p.ph_gofs[ph + 1] <= gq) ++ph;
            uint32_t wv[4] = {0u, 0u, 0u, 0u};
            for (int kb = 0; kb < 4; ++kb) {
                const int g = 4 * (gq - p.ph_gofs[ph]) + kb;
                if (g >= p.ph_tkb[ph]) break;
                const ConvTap T = p.taps[p.ph_tap0[ph] + g / p.CB];
                const uint8_t *bsrc =
                    p.sfb.base + static_cast<int64_t>(T.btap) * p.sfb.tap_pitch + (g % p.CB) * p.sfb.kb_pitch;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int rl = 128 * at + 32 * j + lane;
                    const int r = nt * p.BN + rl;
                    if (rl < p.BN && r < p.sfb.rows)
                        wv[j] |= static_cast<uint32_t>(__ldg(bsrc + (r >> p.sfb.row_shift) * p.sfb.row_pitch)) << (8 * kb);
                }
            }
            *reinterpret_cast<uint4 *>(sSFBc + item * 512 + lane * 16) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        fence_proxy_async_smem();
    }
    if (p.k16) {
        for (int i = threadIdx.x; i < 4096 / 16; i += gemm_threads<KIND>())
            reinterpret_cast<uint4 *>(sZ)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const uint64_t lim = p.timeout_ns;
    const int sf_cols = GA * SPK * (4 * UM + 4 * p.nb_atoms);   // TMEM scale columns per stage

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // the whole warp walks the stages; one elected lane issues the copies
        const bool leader = elect_one();
        uint32_t it = 0;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
            const UnitInfo I = decode_unit<KIND>(p, u);
            KbWalker kw{I.tap0, 0};
            KitWalker kt{0, 0, 0};
            if (KIND == kWgrad) kt.init(p, I.kbase);
            // window boxes: input row of the group's first kernel row at output row 0
            const int wb_h0 = KIND == kWgrad && p.wbox ? I.tap / p.wb_S - p.wb_ph : 0;
            int oq[4], op[4], on[4];             // sub-tile origins
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                oq[i] = I.q0;
                op[i] = I.p0;
                on[i] = I.n0;
                if (KIND == kConv && i > 0 && i < UM) tile_origin(p, I.mt0 + i, oq[i], op[i], on[i]);
            }
            for (int ki = 0; ki < I.nk; ++ki, ++it, s = (s + 1 == S) ? 0 : s + 1, ph ^= (s == 0)) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], ph ^ 1u, lim, abort_flag))) {
                    ok = false;
                    break;
                }
                uint8_t *a_dst = sA + s * a_stage;
                uint8_t *b_dst = sB + s * b_stage;
                if (KIND == kConv) {
                    const int nkb = min(KS, I.tkb - KS * ki);
                    const int nbox = nkb >> lg_wkb;
                    if (leader)
                        mbar_arrive_expect_tx(&full[s],
                                              static_cast<uint32_t>(nbox * (UM * p.a_box_bytes + p.b_box_bytes)));
                    for (int j = 0; j < nbox; ++j) {
                        const ConvTap T = p.taps[kw.tap];
                        const int cx = kw.cb * 32;
                        if (leader) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                if (i >= UM) break;
                                uint8_t *dst = a_dst + i * a_sub_stage + j * 128 * srow;
                                if (NAR)           // 8 pixels x the whole batch (256-byte runs)
                                    tma_load_3d(dst, &p.amap[T.map], &full[s], 0, oq[i] + T.dw, op[i] + T.dh);
                                else if (p.sub > 1)   // slot dimension of extent 1: only slot T.aw is in range
                                    tma_load_5d(dst, &p.amap[T.map], &full[s], cx, -T.aw, oq[i] + T.dw, op[i] + T.dh,
                                                on[i]);
                                else if (p.rows_nfirst)
                                    tma_load_4d(dst, &p.amap[T.map], &full[s], cx, on[i], oq[i] + T.dw, op[i] + T.dh);
                                else
                                    tma_load_4d(dst, &p.amap[T.map], &full[s], cx, oq[i] + T.dw, op[i] + T.dh, on[i]);
                            }
                            tma_load_3d(b_dst + j * p.BN * srow, &p.bmap[0], &full[s], cx, I.col0, T.btap);
                        }
                        kw.advance(p.wkb, p.CB);
                    }
                } else {
                    const int nkit = min(GA, I.nkit - GA * ki);
                    // B: one box over the kit's pixels (one tap), or one box
                    // per (tap, pixel) of a tap group
                    const int bmul = p.ntg > 1 ? (p.wbox ? 1 : I.tig) * p.bqk : 1;
                    if (leader)
                        mbar_arrive_expect_tx(&full[s],
                                              static_cast<uint32_t>(nkit * (p.a_box_bytes + bmul * p.b_box_bytes)));
                    for (int g = 0; g < nkit; ++g) {
                        const int nx = kt.nc * row_bytes;
                        if (leader) {
                            tma_load_4d(a_dst + g * 128 * 4 * kb_bytes, &p.amap[0], &full[s], nx, I.m0 >> rsh,
                                        kt.qg * p.bqk, kt.pp);
                            if (p.ntg == 1) {
                                const ConvTap T = p.taps[I.tap];
                                tma_load_4d(b_dst + g * p.BN * 4 * kb_bytes, &p.bmap[T.map], &full[s], nx,
                                            I.col0 >> rsh, kt.qg * p.bqk + T.dw, kt.pp + T.dh);
                            } else if (p.wbox) {
                                // the group's kernel rows r0.. and all S columns, one box per pixel
                                const int h = p.x_st_h * kt.pp + wb_h0;
                                for (int jq = 0; jq < p.bqk; ++jq)
                                    tma_load_4d(b_dst + g * p.BN * 4 * kb_bytes + jq * p.BN * srow, &p.bmap[0], &full[s],
                                                nx, 0, p.x_st_w * (kt.qg * p.bqk + jq) - p.wb_pw, h);
                            } else {
                                for (int t = 0; t < I.tig; ++t) {
                                    const ConvTap T = p.taps[I.tap + t];
                                    for (int jq = 0; jq < p.bqk; ++jq)
                                        tma_load_4d(b_dst + g * p.BN * 4 * kb_bytes + (jq * p.BN + t * p.cpad) * srow,
                                                    &p.bmap[T.map], &full[s], nx, 0, kt.qg * p.bqk + jq + T.dw,
                                                    kt.pp + T.dh);
                                }
                            }
                        }
                        kt.next(p);
                    }
                }
                __syncwarp();
            }
        }
        if (!ok && leader) {
            // let the copies already in flight land before the CTA exits (a
            // stage whose scale warp gave up never completes; its copy is
            // long done when the short bounded wait below runs out)
            const uint32_t first = it > static_cast<uint32_t>(S) ? it - S : 0u;
            for (uint32_t c = first; c < it; ++c) mbar_wait(&full[c % S], (c / S) & 1u, 20000000ull, nullptr);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // the whole warp walks the stages (so descriptors and TMEM addresses are
        // warp-uniform); one elected lane issues tcgen05.cp / mma / commit
        const bool leader = elect_one();
        uint32_t tcount = 0;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        // descriptors of stage 0, sub-tile 0; other positions add (byte offset
        // >> 4).  k16: no swizzle, 8-row core matrices of 16-byte rows (SBO 128),
        // the second 16 bytes of K at the zero block (LBO = its distance, so an
        // offset added to the start address is taken off the LBO field)
        const uint32_t swz = p.k16 ? static_cast<uint32_t>(kSwizzleNone) : swizzle_of(p.wkb);
        const uint64_t adesc0 = p.k16 ? make_smem_desc(smem_u32(sA), smem_u32(sZ) - smem_u32(sA), 128, swz)
                                      : make_smem_desc(smem_u32(sA), 16, 8 * row_bytes, swz);
        const uint64_t bdesc0 = p.k16 ? make_smem_desc(smem_u32(sB), smem_u32(sZ) - smem_u32(sB), 128, swz)
                                      : make_smem_desc(smem_u32(sB), 16, 8 * row_bytes, swz);
        const uint64_t lbo_step = p.k16 ? (1ull << 16) : 0ull;   // LBO change per 16 bytes of offset
        const uint64_t sfa_desc0 = make_smem_desc(smem_u32(sSFA), 0, 128, kSwizzleNone);
        const uint64_t sfb_desc0 = make_smem_desc(smem_u32(sSFB), 0, 128, kSwizzleNone);
        const uint64_t sfbc_desc0 = make_smem_desc(smem_u32(sSFBc), 0, 128, kSwizzleNone);
        const uint32_t a_sub = (p.a_slab * srow) >> 4, b_sub = (p.b_slab * srow) >> 4;
        const uint32_t a_grp = (128 * 4 * kb_bytes) >> 4, b_grp = (p.BN * 4 * kb_bytes) >> 4;   // 4 K-blocks
        for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
            const UnitInfo I = decode_unit<KIND>(p, u);
            if (I.nk == 0) continue;
            const uint32_t acc = tcount & static_cast<uint32_t>(p.nacc - 1);
            const uint32_t aph = (tcount >> p.lg_nacc) & 1u;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&acc_empty[acc], aph ^ 1u, lim, abort_flag))) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem + acc * UM * p.BN;   // sub-tile i at + i * BN
            // cached B atoms of this column tile
            const int item_base = KIND == kConv ? (I.nt * p.groups + p.ph_gofs[I.ph]) * p.nb_atoms : 0;
            for (int ki = 0; ki < I.nk; ++ki, s = (s + 1 == S) ? 0 : s + 1, ph ^= (s == 0)) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], ph, lim, abort_flag))) {
                    ok = false;
                    break;
                }
                const uint32_t sf_t = tmem + kSfTmemBase + s * sf_cols;     // SFA [group][sub-tile], then SFB
                const uint32_t sfb_t = sf_t + 4 * GA * UM * SPK;
                const int nkb = KIND == kConv ? min(KS, I.tkb - KS * ki) : 4 * min(GA, I.nkit - GA * ki);
                const int ngr = (nkb + 3) >> 2;
                const uint32_t a_s = static_cast<uint32_t>(s * a_stage) >> 4;
                const uint32_t b_s = static_cast<uint32_t>(s * b_stage) >> 4;
                if constexpr (PK != 0) {
                    // K-block kb (one MMA of K = 64) takes its SPK scale bytes
                    // per row from atom kb*SPK/4 at byte (kb*SPK) % 4
                    if (leader) {
                        const int natoms = (nkb * SPK + 3) >> 2;
                        for (int a = 0; a < natoms; ++a) {
                            tc_cp_32x128b_warpx4(sf_t + 4 * a, sfa_desc0 + static_cast<uint64_t>((s * sfa_stage + a * 512) >> 4));
                            tc_cp_32x128b_warpx4(sfb_t + 4 * a, sfb_desc0 + static_cast<uint64_t>((s * sfb_stage + a * 512) >> 4));
                        }
                        for (int kb = 0; kb < nkb; ++kb) {
                            const uint32_t g = static_cast<uint32_t>(kb >> 2), k4 = static_cast<uint32_t>(kb & 3);
                            const uint32_t j = k4 >> lg_wkb;
                            const uint32_t within = k4 & static_cast<uint32_t>(p.wkb - 1);
                            const uint32_t bo = b_s + g * b_grp + j * b_sub + within * 2;
                            const uint32_t ao = a_s + g * a_grp + j * a_sub + within * 2;
                            const uint32_t at = static_cast<uint32_t>(kb * SPK) >> 2, sid = static_cast<uint32_t>(kb * SPK) & 3u;
                            if (PK == 2)
                                tc_mma_nvf4(d_tmem, adesc0 + ao, bdesc0 + bo, p.idesc, sf_t + 4 * at, sfb_t + 4 * at,
                                            (ki > 0 || kb > 0) ? 1u : 0u);
                            else
                                tc_mma_mxf4(d_tmem, adesc0 + ao, bdesc0 + bo, p.idesc | (sid << 29) | (sid << 4),
                                            (sf_t + 4 * at) | (sid << 30), (sfb_t + 4 * at) | (sid << 30),
                                            (ki > 0 || kb > 0) ? 1u : 0u);
                        }
                        tc_commit(&empty[s]);
                    }
                    __syncwarp();
                    continue;
                }
                if (leader) {
                    for (int g = 0; g < ngr; ++g) {
                        for (int i = 0; i < UM; ++i)
                            tc_cp_32x128b_warpx4(sf_t + 4 * (g * UM + i),
                                                 sfa_desc0 + static_cast<uint64_t>((s * sfa_stage + (g * UM + i) * 512) >> 4));
                        for (int a = 0; a < p.nb_atoms; ++a) {
                            const uint64_t src =
                                (KIND == kConv && p.sfb_cached)
                                    ? sfbc_desc0 + static_cast<uint64_t>(((item_base + (ki * GA + g) * p.nb_atoms + a) * 512) >> 4)
                                    : sfb_desc0 + static_cast<uint64_t>((s * sfb_stage + (g * p.nb_atoms + a) * 512) >> 4);
                            tc_cp_32x128b_warpx4(sfb_t + 4 * (g * p.nb_atoms + a), src);
                        }
                    }
                    for (int kb = 0; kb < nkb; ++kb) {
                        const uint32_t g = static_cast<uint32_t>(kb >> 2), k4 = static_cast<uint32_t>(kb & 3);
                        const uint32_t j = k4 >> lg_wkb;                       // sub-tile within the group
                        const uint32_t within = k4 & static_cast<uint32_t>(p.wkb - 1);
                        const uint32_t bo = b_s + g * b_grp + j * b_sub + within * 2;
                        for (int i = 0; i < UM; ++i) {
                            const uint32_t ao = a_s + ((i * a_sub_stage) >> 4) + g * a_grp + j * a_sub + within * 2;
                            tc_mma_mxf8f6f4(d_tmem + i * p.BN, adesc0 + ao - ao * lbo_step, bdesc0 + bo - bo * lbo_step,
                                            p.idesc | (k4 << 29) | (k4 << 4),
                                            (sf_t + 4 * (g * UM + i)) | (k4 << 30), (sfb_t + 4 * g * p.nb_atoms) | (k4 << 30),
                                            (ki > 0 || kb > 0) ? 1u : 0u);
                        }
                    }
                    tc_commit(&empty[s]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (leader) tc_commit(&acc_full[acc]);
            __syncwarp();
            ++tcount;
        }
    } else if (sf_warp_index(warp) >= 0 && sf_warp_index(warp) < (p.nsf > 0 ? p.nsf : min(kNumSfWarps, S))) {
        // ------------------------------------------------------------ scale-factor gather
        // scale warp w handles the stages whose global index is w modulo nsf.
        // nsf <= S: a warp's consecutive stages are at most S apart, so when
        // it waits for slot s it is never two phases ahead of the consumer
        // (a parity wait cannot tell phase r from phase r - 2)
        const int nsf = p.nsf > 0 ? p.nsf : min(kNumSfWarps, S);
        const int sfw = sf_warp_index(warp);
        uint32_t it = 0;             // global index of the first stage of the unit
        uint32_t gnext = static_cast<uint32_t>(sfw);   // global index of this warp's next stage
        int s = sfw % S;
        uint32_t ph = static_cast<uint32_t>(sfw / S) & 1u;
        bool ok = true;
        const bool skip_b = KIND == kConv && p.sfb_cached;
        // CONV: this lane's rows lane + 32 j, decoded once
        uint32_t rdec[4] = {0u, 0u, 0u, 0u};
        if (ROWDEC) {
#pragma unroll
            for (int j = 0; j < 4; ++j) rdec[j] = conv_row_packed(p, lane + 32 * j);
        }
        for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
            const UnitInfo I = decode_unit<KIND>(p, u);
            const uint32_t it_unit = it;
            it += static_cast<uint32_t>(I.nk);
            if (gnext >= it) continue;
            const int first = static_cast<int>(gnext - it_unit);
            // A rows of this lane: m = lane + 32 j of sub-tile i
            int ra_h[4], ra_w[4], ra_off[4], ra_aw[4];
            bool ra_ok[4];
            auto set_rows = [&](int i) {
                if (KIND == kWgrad && SFV4) {
                    // this lane's A byte: row group (lane >> 2) & 3 (lanes 0-15)
                    const int k = I.m0 + 32 * ((lane >> 2) & 3);
                    ra_ok[0] = lane < 16 && k < p.sfa.rows;
                    ra_off[0] = (k >> 5) * p.sfa.row_pitch;
                    return;
                }
                int q0 = I.q0, p0 = I.p0, n0 = I.n0;
                if (KIND == kConv && i > 0) tile_origin(p, I.mt0 + i, q0, p0, n0);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int m = lane + 32 * j;
                    if (KIND == kConv) {
                        const uint32_t d = ROWDEC ? rdec[j] : conv_row_packed(p, m);
                        const int aw = d & 0xFF, iq = (d >> 8) & 0xFF, ip = (d >> 16) & 0xFF, in = (d >> 24) & 0x7F;
                        const int q = q0 + iq, pr = p0 + ip, n = n0 + in;
                        ra_ok[j] = !(d >> 31) && p.sub * q + aw < p.ph_Qe[I.ph] && pr < p.ph_Pe[I.ph] && n < p.Ne;
                        ra_h[j] = p.a_st_h * pr;
                        ra_w[j] = p.a_st_w * q;
                        ra_aw[j] = aw;
                        ra_off[j] = (n >> p.sfa.row_shift) * p.sfa.row_pitch;
                    } else {
                        const int k = I.m0 + m;
                        ra_ok[j] = k < p.sfa.rows;
                        ra_h[j] = 0;
                        ra_w[j] = 0;
                        ra_aw[j] = 0;
                        ra_off[j] = (k >> p.sfa.row_shift) * p.sfa.row_pitch;
                    }
                }
            };
            // NAR, sf_pix: per sub-tile i, this lane's pixel (lane % 8) as a
            // scale row and column before the tap offset (a row far out of
            // range for pixels past the output) and its batch block offset
            int np_h[4] = {0, 0, 0, 0}, np_w[4] = {0, 0, 0, 0}, np_o[4] = {0, 0, 0, 0};
            const bool nar_pix = KIND == kConv && NAR && p.sf_pix;
            if (nar_pix) {
                const int pi = lane & 7;
                const int ip = static_cast<int>(p.fd_bq.div(static_cast<uint32_t>(pi)));
                const int iq = pi - ip * p.bq;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (i >= UM) break;
                    int q0 = I.q0, p0 = I.p0, n0 = I.n0;
                    if (i > 0) tile_origin(p, I.mt0 + i, q0, p0, n0);
                    const int q = q0 + iq, pr = p0 + ip;
                    const bool okp = q < p.ph_Qe[I.ph] && pr < p.ph_Pe[I.ph] && n0 < p.Ne;
                    np_h[i] = okp ? p.a_st_h * pr : -(1 << 20);
                    np_w[i] = p.a_st_w * q;
                    np_o[i] = (n0 >> 5) * p.sfa.row_pitch;
                }
            } else {
                set_rows(0);
            }
            // B rows of this lane: col0 + 128 at + 32 j + lane
            // (WGRAD: with tap groups a B row is (tap, channel) and carries
            // its tap's pixel offset; otherwise every row has the unit's tap)
            int rb_off[2][4], rb_dh[2][4], rb_dw[2][4];
            bool rb_ok[2][4];
            if (KIND == kWgrad && SFV4) {
                // this lane's B bytes: with 16-row groups, group 2 ((lane >> 3) & 3) +
                // ((lane >> 2) & 1) of atom 0 and of atom 1; with 32-row groups,
                // group (lane >> 2) & 3 of atom lane >> 4 (one byte)
#pragma unroll
                for (int at = 0; at < 2; ++at) {
                    const int atom = p.sq16 ? at : lane >> 4;
                    const int rl = p.sq16 ? 128 * at + 32 * ((lane >> 3) & 3) + 16 * ((lane >> 2) & 1)
                                          : 128 * atom + 32 * ((lane >> 2) & 3);
                    const int t = p.ntg > 1 ? static_cast<int>(p.fd_cpad.div(rl)) : 0;
                    const int r = I.col0 + rl - t * p.cpad;
                    rb_ok[at][0] = atom < p.nb_atoms && rl < p.BN && r < p.sfb.rows && t < I.tig;
                    rb_off[at][0] = (r >> 5) * p.sfb.row_pitch;
                    const ConvTap T = p.taps[I.tap + (rb_ok[at][0] ? t : 0)];
                    rb_dh[at][0] = T.sf_dh;
                    rb_dw[at][0] = T.sf_dw;
                }
            } else {
#pragma unroll
            for (int at = 0; at < 2; ++at)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int rl = 128 * at + 32 * j + lane;
                    int r = I.col0 + rl, t = 0;
                    if (KIND == kWgrad && p.ntg > 1) {
                        t = static_cast<int>(p.fd_cpad.div(rl));
                        r = rl - t * p.cpad;
                    }
                    rb_ok[at][j] = at < p.nb_atoms && rl < p.BN && r < p.sfb.rows && (KIND == kConv || t < I.tig);
                    rb_off[at][j] = (r >> p.sfb.row_shift) * p.sfb.row_pitch;
                    if (KIND == kWgrad) {
                        const ConvTap T = p.taps[I.tap + (rb_ok[at][j] ? t : 0)];
                        rb_dh[at][j] = T.sf_dh;
                        rb_dw[at][j] = T.sf_dw;
                    } else {
                        rb_dh[at][j] = rb_dw[at][j] = 0;
                    }
                }
            }
            KbWalker kw{I.tap0, 0};
            KitWalker kt{0, 0, 0};
            if (KIND == kConv) kw.advance(KS * first, p.CB);
            else kt.init(p, I.kbase + GA * first);
            for (int ki = first; ki < I.nk; ki += nsf) {
                // one group of 4 K-blocks (one scale atom per operand) at a
                // time: gather into registers, then store; the stage slot is
                // awaited before the first store (the loads of the first
                // group are already in flight by then)
                const int ngr = KIND == kConv ? (min(KS, I.tkb - KS * ki) + 3) >> 2 : min(GA, I.nkit - GA * ki);
                const int nkb = KIND == kConv ? min(KS, I.tkb - KS * ki) : 4 * ngr;
                KbWalker k2 = kw;
                KitWalker k3 = kt;
                bool slot = false;
                for (int g = 0; g < GA && ok; ++g) {
                  const KbWalker kg = k2;                 // start of the group (each sub-tile walks it)
                  // NAR, sf_pix: scale offsets of this lane's K-block (lane / 8,
                  // one tap each) of the group, read uniformly (out of range
                  // past the stage's K-blocks)
                  int tdh = -(1 << 20), tdw = 0;
                  if (nar_pix) {
#pragma unroll
                      for (int kb = 0; kb < 4; ++kb)
                          if (4 * g + kb < nkb) {
                              const ConvTap T = p.taps[kg.tap + kb];
                              if (kb == (lane >> 3)) {
                                  tdh = T.sf_dh;
                                  tdw = T.sf_dw;
                              }
                          }
                  }
                  for (int i = 0; i < UM; ++i) {
                    if constexpr (KIND == kConv && PK != 0) {
                        // SPK scales per row and K-block (2 E8M0 for MXFP4, 4
                        // UE4M3 for NVFP4): K-block kb fills bytes (kb*SPK) % 4
                        // .. of atom kb*SPK/4; blocks past the row's last read
                        // as 0 (their codes are TMA zero fill)
                        uint32_t na[4][4] = {}, nb[4][4] = {};   // [atom][row j]
                        if (g < ngr && p.sf_vec4) {
                            // whole atoms with one aligned 32-bit load per row:
                            // atom a = K-blocks a*4/SPK .. of one tap, scale
                            // blocks SPK*cb .. SPK*cb + 3 adjacent (host check)
#pragma unroll
                            for (int a = 0; a < SPK; ++a) {
                                if (4 * g + a * (4 / SPK) >= nkb) break;
                                const ConvTap T = p.taps[k2.tap];
                                const int cb = k2.cb;
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const int hh = ra_h[j] + T.sf_dh, ww = ra_w[j] + T.sf_dw;
                                    if (ra_ok[j] && ra_aw[j] == T.aw && hh >= 0 && hh < p.sfa.H && ww >= 0 && ww < p.sfa.W)
                                        na[a][j] = __ldg(reinterpret_cast<const uint32_t *>(
                                            p.sfa.base + (static_cast<int64_t>(hh) * p.sfa.W + ww) * p.sfa.pix_pitch + ra_off[j] +
                                            SPK * cb));
                                }
                                const uint8_t *bsrc = p.sfb.base + static_cast<int64_t>(T.btap) * p.sfb.tap_pitch;
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    if (!rb_ok[0][j]) continue;
                                    if (p.sfb.kb_pitch == 1) {
                                        nb[a][j] = __ldg(reinterpret_cast<const uint32_t *>(bsrc + rb_off[0][j] + SPK * cb));
                                    } else {   // the B scales of consecutive blocks are kb_pitch apart
                                        uint32_t w = 0u;
#pragma unroll
                                        for (int q = 0; q < 4; ++q)
                                            w |= static_cast<uint32_t>(__ldg(bsrc + rb_off[0][j] + (SPK * cb + q) * p.sfb.kb_pitch)) << (8 * q);
                                        nb[a][j] = w;
                                    }
                                }
                                k2.advance(4 / SPK, p.CB);
                            }
                        } else if (g < ngr) {
#pragma unroll
                            for (int kb = 0; kb < 4; ++kb) {
                                if (4 * g + kb >= nkb) break;
                                const ConvTap T = p.taps[k2.tap];
                                const int cb = k2.cb;
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const int hh = ra_h[j] + T.sf_dh, ww = ra_w[j] + T.sf_dw;
                                    if (ra_ok[j] && ra_aw[j] == T.aw && hh >= 0 && hh < p.sfa.H && ww >= 0 && ww < p.sfa.W) {
                                        // scale block SPK*cb + q along K, kb_pitch bytes apart
                                        const uint8_t *src = p.sfa.base + (static_cast<int64_t>(hh) * p.sfa.W + ww) * p.sfa.pix_pitch +
                                                             ra_off[j];
                                        uint32_t w = 0u;
#pragma unroll
                                        for (int q = 0; q < SPK; ++q)
                                            if (SPK * cb + q < p.sfa.nblk)
                                                w |= static_cast<uint32_t>(__ldg(src + (SPK * cb + q) * p.sfa.kb_pitch)) << (8 * q);
                                        na[(kb * SPK) >> 2][j] |= w << (8 * ((kb * SPK) & 3));
                                    }
                                }
                                const uint8_t *bsrc = p.sfb.base + static_cast<int64_t>(T.btap) * p.sfb.tap_pitch;
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    if (!rb_ok[0][j]) continue;
                                    uint32_t w = 0u;
#pragma unroll
                                    for (int q = 0; q < SPK; ++q)
                                        if (SPK * cb + q < p.sfb.nblk)
                                            w |= static_cast<uint32_t>(__ldg(bsrc + rb_off[0][j] + (SPK * cb + q) * p.sfb.kb_pitch)) << (8 * q);
                                    nb[(kb * SPK) >> 2][j] |= w << (8 * ((kb * SPK) & 3));
                                }
                                k2.advance(1, p.CB);
                            }
                        }
                        if (!slot) {
                            if (!mbar_wait(&empty[s], ph ^ 1u, lim, abort_flag)) {
                                ok = false;
                                break;
                            }
                            slot = true;
                        }
#pragma unroll
                        for (int a = 0; a < SPK; ++a) {
                            *reinterpret_cast<uint4 *>(sSFA + s * sfa_stage + (g * SPK + a) * 512 + lane * 16) =
                                make_uint4(na[a][0], na[a][1], na[a][2], na[a][3]);
                            *reinterpret_cast<uint4 *>(sSFB + s * sfb_stage + (g * SPK + a) * 512 + lane * 16) =
                                make_uint4(nb[a][0], nb[a][1], nb[a][2], nb[a][3]);
                        }
                        continue;
                    }
                    if (UM > 1) {
                        if (!nar_pix) set_rows(i);
                        k2 = kg;
                    }
                    const bool gb = i == 0 && !skip_b;      // B atoms: once per group
                    uint32_t wa[4] = {0u, 0u, 0u, 0u};      // [row j]
                    uint32_t wb[2][4] = {};                 // [atom][row j]
                    if (g < ngr) {
                        if (KIND == kConv && SFV4) {
                            // one tap, channel blocks cb..cb+3: one 32-bit load per row
                            const ConvTap T = p.taps[k2.tap];
                            const int cb = k2.cb;
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int hh = ra_h[j] + T.sf_dh, ww = ra_w[j] + T.sf_dw;
                                if (ra_ok[j] && ra_aw[j] == T.aw && hh >= 0 && hh < p.sfa.H && ww >= 0 && ww < p.sfa.W)
                                    wa[j] = __ldg(reinterpret_cast<const uint32_t *>(
                                        p.sfa.base + (static_cast<int64_t>(hh) * p.sfa.W + ww) * p.sfa.pix_pitch +
                                        ra_off[j] + cb));
                            }
                            if (gb) {
                                const uint8_t *bsrc = p.sfb.base + static_cast<int64_t>(T.btap) * p.sfb.tap_pitch + cb;
#pragma unroll
                                for (int at = 0; at < 2; ++at)
#pragma unroll
                                    for (int j = 0; j < 4; ++j)
                                        if (rb_ok[at][j])
                                            wb[at][j] = __ldg(reinterpret_cast<const uint32_t *>(bsrc + rb_off[at][j]));
                            }
                            k2.advance(4, p.CB);
                        } else if (KIND == kConv && NAR && p.sf_pix) {
                            // 8 pixels x 16 batch rows, one scale byte per pixel
                            // and tap: lane l loads pixel l % 8 of K-block l / 8
                            // (one tap each, CB = 1); row m takes pixel m / 16
                            int bh = np_h[0], bw = np_w[0], bo = np_o[0];
#pragma unroll
                            for (int t = 1; t < 4; ++t)
                                if (t == i) {
                                    bh = np_h[t];
                                    bw = np_w[t];
                                    bo = np_o[t];
                                }
                            const int hh = bh + tdh, ww = bw + tdw;
                            uint32_t v = 0u;
                            if (hh >= 0 && hh < p.sfa.H && ww >= 0 && ww < p.sfa.W)
                                v = __ldg(p.sfa.base + (static_cast<int64_t>(hh) * p.sfa.W + ww) * p.sfa.pix_pitch + bo);
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int pix = (lane >> 4) + 2 * j;
                                uint32_t w = 0u;
#pragma unroll
                                for (int kb = 0; kb < 4; ++kb) w |= __shfl_sync(0xFFFFFFFFu, v, pix + 8 * kb) << (8 * kb);
                                wa[j] = w;
                            }
                            for (int kb = 0; kb < 4 && 4 * g + kb < nkb; ++kb) {
                                if (gb) {
                                    const ConvTap T = p.taps[k2.tap];
                                    const uint8_t *bsrc = p.sfb.base + static_cast<int64_t>(T.btap) * p.sfb.tap_pitch;
#pragma unroll
                                    for (int at = 0; at < 2; ++at)
#pragma unroll
                                        for (int j = 0; j < 4; ++j)
                                            if (rb_ok[at][j])
                                                wb[at][j] |= static_cast<uint32_t>(__ldg(bsrc + rb_off[at][j])) << (8 * kb);
                                }
                                k2.advance(1, p.CB);
                            }
                        } else if (KIND == kConv) {
                            for (int kb = 0; kb < 4 && 4 * g + kb < nkb; ++kb) {
                                const ConvTap T = p.taps[k2.tap];
                                const int cb = k2.cb;
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const int hh = ra_h[j] + T.sf_dh, ww = ra_w[j] + T.sf_dw;
                                    if (ra_ok[j] && ra_aw[j] == T.aw && hh >= 0 && hh < p.sfa.H && ww >= 0 &&
                                        ww < p.sfa.W)
                                        wa[j] |= static_cast<uint32_t>(__ldg(
                                                     p.sfa.base +
                                                     (static_cast<int64_t>(hh) * p.sfa.W + ww) * p.sfa.pix_pitch +
                                                     ra_off[j] + cb * p.sfa.kb_pitch))
                                                 << (8 * kb);
                                }
                                if (gb) {
                                    const uint8_t *bsrc =
                                        p.sfb.base + static_cast<int64_t>(T.btap) * p.sfb.tap_pitch + cb * p.sfb.kb_pitch;
#pragma unroll
                                    for (int at = 0; at < 2; ++at)
#pragma unroll
                                        for (int j = 0; j < 4; ++j)
                                            if (rb_ok[at][j])
                                                wb[at][j] |= static_cast<uint32_t>(__ldg(bsrc + rb_off[at][j])) << (8 * kb);
                                }
                                k2.advance(1, p.CB);
                            }
                        } else if (SFV4) {
                            // lane: K-block lane & 3; A row group (lane >> 2) & 3
                            // (lanes 0-15); B 16-row group of each atom as above
                            const int kbl = lane & 3;
                            const int q = k3.qg * p.bqk + (kbl >> lg_wkb);
                            const int nb = k3.nc * p.wkb + (kbl & (p.wkb - 1));
                            uint32_t va = 0u, vb[2] = {0u, 0u};
                            if (q < p.Q) {
                                const int64_t pix = static_cast<int64_t>(k3.pp) * p.Q + q;
                                if (ra_ok[0])
                                    va = __ldg(p.sfa.base + pix * p.sfa.pix_pitch + nb * p.sfa.kb_pitch + ra_off[0]);
#pragma unroll
                                for (int at = 0; at < 2; ++at) {
                                    if (at == 1 && !p.sq16) break;
                                    const int hh = p.x_st_h * k3.pp + rb_dh[at][0], ww = p.x_st_w * q + rb_dw[at][0];
                                    if (rb_ok[at][0] && hh >= 0 && hh < p.sfb.H && ww >= 0 && ww < p.sfb.W)
                                        vb[at] = __ldg(p.sfb.base +
                                                       (static_cast<int64_t>(hh) * p.sfb.W + ww) * p.sfb.pix_pitch +
                                                       nb * p.sfb.kb_pitch + rb_off[at][0]);
                                }
                            }
                            va <<= 8 * kbl;
                            vb[0] <<= 8 * kbl;
                            vb[1] <<= 8 * kbl;
#pragma unroll
                            for (int x = 1; x <= 2; x <<= 1) {
                                va |= __shfl_xor_sync(0xFFFFFFFFu, va, x);
                                vb[0] |= __shfl_xor_sync(0xFFFFFFFFu, vb[0], x);
                                if (p.sq16) vb[1] |= __shfl_xor_sync(0xFFFFFFFFu, vb[1], x);
                            }
                            if (!p.sq16) vb[1] = vb[0];
                            // row lane + 32 j of B atom `at`: 16-row group 2 j + (lane >> 4)
                            // of vb[at], or 32-row group j of atom at in vb[0]
                            const int b0 = p.sq16 ? 4 * (lane >> 4) : 0, b1 = p.sq16 ? b0 : 16;
                            const int bstep = p.sq16 ? 8 : 4;
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                wa[j] = __shfl_sync(0xFFFFFFFFu, va, 4 * j);
                                wb[0][j] = __shfl_sync(0xFFFFFFFFu, vb[0], b0 + bstep * j);
                                wb[1][j] = __shfl_sync(0xFFFFFFFFu, vb[1], b1 + bstep * j);
                            }
                            k3.next(p);
                        } else {
                            for (int kb = 0; kb < 4; ++kb) {
                                const int q = k3.qg * p.bqk + (kb >> lg_wkb);
                                const int nb = k3.nc * p.wkb + (kb & (p.wkb - 1));
                                if (q >= p.Q) continue;
                                const uint8_t *asrc = p.sfa.base +
                                                      (static_cast<int64_t>(k3.pp) * p.Q + q) * p.sfa.pix_pitch +
                                                      nb * p.sfa.kb_pitch;
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    if (ra_ok[j]) wa[j] |= static_cast<uint32_t>(__ldg(asrc + ra_off[j])) << (8 * kb);
                                const int h0 = p.x_st_h * k3.pp, w0 = p.x_st_w * q;
                                if (p.ntg == 1) {
                                    // every row has the unit's tap: one pixel per K-block
                                    const int hh = h0 + rb_dh[0][0], ww = w0 + rb_dw[0][0];
                                    if (hh < 0 || hh >= p.sfb.H || ww < 0 || ww >= p.sfb.W) continue;
                                    const uint8_t *bsrc = p.sfb.base +
                                                          (static_cast<int64_t>(hh) * p.sfb.W + ww) * p.sfb.pix_pitch +
                                                          nb * p.sfb.kb_pitch;
#pragma unroll
                                    for (int at = 0; at < 2; ++at)
#pragma unroll
                                        for (int j = 0; j < 4; ++j)
                                            if (rb_ok[at][j])
                                                wb[at][j] |= static_cast<uint32_t>(__ldg(bsrc + rb_off[at][j])) << (8 * kb);
                                    continue;
                                }
#pragma unroll
                                for (int at = 0; at < 2; ++at)
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        const int hh = h0 + rb_dh[at][j], ww = w0 + rb_dw[at][j];
                                        if (rb_ok[at][j] && hh >= 0 && hh < p.sfb.H && ww >= 0 && ww < p.sfb.W)
                                            wb[at][j] |= static_cast<uint32_t>(__ldg(
                                                             p.sfb.base +
                                                             (static_cast<int64_t>(hh) * p.sfb.W + ww) * p.sfb.pix_pitch +
                                                             nb * p.sfb.kb_pitch + rb_off[at][j]))
                                                         << (8 * kb);
                                    }
                            }
                            k3.next(p);
                        }
                    }
                    if (!slot) {
                        if (!mbar_wait(&empty[s], ph ^ 1u, lim, abort_flag)) {
                            ok = false;
                            break;
                        }
                        slot = true;
                    }
                    *reinterpret_cast<uint4 *>(sSFA + s * sfa_stage + (g * UM + i) * 512 + lane * 16) =
                        make_uint4(wa[0], wa[1], wa[2], wa[3]);
                    if (gb) {
                        *reinterpret_cast<uint4 *>(sSFB + s * sfb_stage + (g * p.nb_atoms) * 512 + lane * 16) =
                            make_uint4(wb[0][0], wb[0][1], wb[0][2], wb[0][3]);
                        if (p.nb_atoms > 1)
                            *reinterpret_cast<uint4 *>(sSFB + s * sfb_stage + (g * p.nb_atoms + 1) * 512 + lane * 16) =
                                make_uint4(wb[1][0], wb[1][1], wb[1][2], wb[1][3]);
                    }
                  }
                }
                if (!ok) break;
                if (KIND == kConv) kw.advance(KS * nsf, p.CB);
                else
                    for (int step = 0; step < GA * nsf; ++step) kt.next(p);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[s]);
                gnext += nsf;
                s += nsf;
                while (s >= S) {
                    s -= S;
                    ph ^= 1u;
                }
            }
        }
    } else if ((warp >= 4 && warp < 8) || (KIND == kConv && warp >= 12)) {
        // ------------------------------------------------------------ epilogue
        const int qd = warp & 3;               // TMEM lane quadrant of this warp
        const int m = qd * 32 + lane;
        const int team = warp >= 12 ? 1 : 0;   // team t: accumulators t, t + 2 (tiles t modulo 2)
        // one team for the depth-to-space stores (their half-sector writes
        // measured slower with twice as many in flight)
        const int nteams = KIND == kConv && p.nacc >= 2 && !p.d2s ? 2 : 1;
        uint32_t tcount = 0;
        uint32_t ep_round = 0;                 // ep_stage: staging rounds of this team (buffer, barrier phase)
        bool ep_fail = false;
        const uint32_t edec0 = ROWDEC ? conv_row_packed(p, m) : 0u;   // this thread's row, decoded once

        for (int u = blockIdx.x; u < p.num_units && team < nteams && !ep_fail; u += gridDim.x) {
            const UnitInfo I = decode_unit<KIND>(p, u);
            // output row of this thread in sub-tile i
            bool row_ok;
            int64_t row_off;
            auto set_row = [&](int i) {
                if (KIND == kConv) {
                    int q0 = I.q0, p0 = I.p0, n0 = I.n0;
                    if (i > 0) tile_origin(p, I.mt0 + i, q0, p0, n0);
                    const uint32_t edec = ROWDEC ? edec0 : conv_row_packed(p, m);
                    const int e_aw = edec & 0xFF, e_iq = (edec >> 8) & 0xFF, e_ip = (edec >> 16) & 0xFF;
                    const int e_in = (edec >> 24) & 0x7F;
                    const int q = p.sub * (q0 + e_iq) + e_aw, pr = p0 + e_ip, n = n0 + e_in;
                    row_ok = !(edec >> 31) && q < p.ph_Qe[I.ph] && pr < p.ph_Pe[I.ph] && n < p.Ne;
                    row_off = p.ph_out_base[I.ph] + n * p.os_n + pr * p.os_p + q * p.os_q;
                } else {
                    const int k = I.m0 + m;
                    row_ok = k < p.Mrows;
                    row_off = p.out_base + I.split * p.split_pitch + k * p.os_m + (p.ntg == 1 ? p.taps[I.tap].btap : 0);
                }
            };
            const bool tap_cols = KIND == kWgrad && p.ntg > 1;   // columns are (tap, channel)
            if (I.nk == 0) {
                if (team != 0 || QOUT) continue;   // (a forward tile always has K-blocks)
                for (int i = 0; i < UM; ++i) {
                    set_row(i);
                    if (row_ok)
                        for (int n = 0; n < p.BN; ++n) {
                            if (KIND == kConv && p.d2s) {
                                const int cs = I.col0 + n;
                                const int ph = static_cast<int>(p.fd_cpad.div(cs));
                                if (cs < p.Ncols) p.out[row_off + (cs - ph * p.cpad) * p.os_c + p.d2s_off[ph]] = 0.0f;
                            } else if (tap_cols) {
                                const int t = static_cast<int>(p.fd_cpad.div(n)), c = n - t * p.cpad;
                                if (t < I.tig && c < p.Ncols) p.out[row_off + c * p.os_c + p.taps[I.tap + t].btap] = 0.0f;
                            } else if (I.col0 + n < p.Ncols) {
                                p.out[row_off + (I.col0 + n) * p.os_c] = 0.0f;
                            }
                        }
                }
                continue;
            }
            if (nteams == 2 && static_cast<int>(tcount & 1u) != team) {
                ++tcount;
                continue;
            }
            const uint32_t acc = tcount & static_cast<uint32_t>(p.nacc - 1);
            const uint32_t aph = (tcount >> p.lg_nacc) & 1u;
            if (!mbar_wait(&acc_full[acc], aph, lim, abort_flag)) break;
            tc_fence_after();
            // 32 columns at a time (one TMEM load, one wait); the accumulators
            // are released after the last load of the last sub-tile, before
            // its global stores, so the MMA issuer can start the next unit on
            // them.  The loop body is kept small: it runs once per 32 columns
            // of every sub-tile, next to the code of the other roles.
            for (int i = 0; i < UM; ++i) {
                set_row(i);
                const uint32_t t_row = tmem + (static_cast<uint32_t>(qd * 32) << 16) + (acc * UM + i) * p.BN;
                if constexpr (KIND == kConv && QOUT) {
                    // next-layer pixel and batch index of this row
                    int q0 = I.q0, p0 = I.p0, n0 = I.n0;
                    if (i > 0) tile_origin(p, I.mt0 + i, q0, p0, n0);
                    const uint32_t edec = ROWDEC ? edec0 : conv_row_packed(p, m);
                    const int e_iq = (edec >> 8) & 0xFF, e_ip = (edec >> 16) & 0xFF, e_in = (edec >> 24) & 0x7F;
                    const int qpix = (p0 + e_ip) * p.ph_Qe[0] + (q0 + e_iq);
                    for (int c0 = 0; c0 < p.BN; c0 += 32) {
                        uint32_t r[32];
                        tc_ld_32x32b_x32(t_row + c0, r);
                        tc_wait_ld();
                        if (i + 1 == UM && c0 + 32 >= p.BN) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&acc_empty[acc]);
                        }
                        if (I.col0 + c0 < p.Ncols)
                            qout_chunk(p, r, row_ok, qpix, n0 + e_in, I.col0 + c0, sTr + (team * 4 + qd) * (32 * 9), lane);
                    }
                    continue;
                }
                if (KIND == kConv && NAR && !QOUT && p.ep_stage) {
                    // batch-first rows: row m is batch m % 16 at pixel m / 16
                    // (q0 + m / 16); the team writes the tile as [n][column][q]
                    // and warp qd stores batch rows 4 qd .. 4 qd + 3, each
                    // (n, channel) as two 16-byte runs of 4 q
                    int q0 = I.q0, p0 = I.p0, n0 = I.n0;
                    if (i > 0) tile_origin(p, I.mt0 + i, q0, p0, n0);
                    for (int c0 = 0; c0 < p.BN; c0 += 32) {
                        uint32_t r[32];
                        tc_ld_32x32b_x32(t_row + c0, r);
                        tc_wait_ld();
                        if (i + 1 == UM && c0 + 32 >= p.BN) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&acc_empty[acc]);
                        }
                        float *stg = sEp + (team * 2 + (ep_round & 1u)) * (16 * 260);
                        float *w = stg + (m & 15) * 260 + (m >> 4);
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) w[jj * 8] = __uint_as_float(r[jj]);
                        // the four warps of the team have written the tile (a
                        // buffer is rewritten two rounds later, after every
                        // warp has passed the next round's barrier, i.e. has
                        // finished reading it)
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ep_bar[team]);
                        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&ep_bar[team], ep_round & 1u, lim, abort_flag))) {
                            ep_fail = true;
                            break;
                        }
                        ++ep_round;
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            const int idx = t * 32 + lane;
                            const int nn = qd * 4 + (idx >> 6), k = (idx >> 1) & 31, half = idx & 1;
                            const float4 v = *reinterpret_cast<const float4 *>(stg + nn * 260 + k * 8 + half * 4);
                            const int n = n0 + nn, col = I.col0 + c0 + k, q = q0 + half * 4;
                            if (n < p.Ne && col < p.Ncols && q < p.ph_Qe[0] && p0 < p.ph_Pe[0])
                                *reinterpret_cast<float4 *>(p.out + n * p.os_n + col * p.os_c + p0 * p.os_p + q) = v;
                        }
                    }
                    if (ep_fail) break;
                    continue;
                }
                float *orow = p.out + row_off;
                if (KIND == kConv && p.d2s == 2) {
                    // 16 channels of a phase pair (aw = 0, 1) per pass: column
                    // pa and pa + cpad, stored together as 8-byte pairs
                    for (int c0 = 0; c0 < p.BN; c0 += 32) {
                        uint32_t r[32];
                        const int q = c0 >> 5, nblk = p.cpad >> 4;   // 16-channel blocks of a phase
                        const int pp = q / nblk;
                        const int pc = (q - pp * nblk) << 4;
                        const int pa = 2 * pp * p.cpad + pc;
                        tc_ld_32x32b_x16p(t_row + pa, r);
                        tc_ld_32x32b_x16p(t_row + pa + p.cpad, r + 16);
                        tc_wait_ld();
                        if (i + 1 == UM && c0 + 32 >= p.BN) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&acc_empty[acc]);
                        }
                        const int n0 = I.col0 + pa;
                        if (row_ok && n0 < p.Ncols) {
                            const int ph = static_cast<int>(p.fd_cpad.div(n0));
                            float *op = orow + static_cast<int64_t>(pc) * p.os_c + p.d2s_off[ph];
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj)
                                *reinterpret_cast<float2 *>(op + jj * p.os_c) =
                                    make_float2(__uint_as_float(r[jj]), __uint_as_float(r[16 + jj]));
                        }
                    }
                    continue;
                }
                for (int c0 = 0; c0 < p.BN; c0 += 32) {
                    uint32_t r[32];
                    tc_ld_32x32b_x32(t_row + c0, r);
                    tc_wait_ld();
                    if (i + 1 == UM && c0 + 32 >= p.BN) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&acc_empty[acc]);
                    }
                    if (KIND == kConv && p.d2s) {
                        // 16 columns at a time: one phase, consecutive channels
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int n0 = I.col0 + c0 + 16 * h;
                            if (!row_ok || n0 >= p.Ncols) continue;
                            const int ph = static_cast<int>(p.fd_cpad.div(n0));
                            float *op = orow + static_cast<int64_t>(n0 - ph * p.cpad) * p.os_c + p.d2s_off[ph];
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) op[jj * p.os_c] = __uint_as_float(r[16 * h + jj]);
                        }
                        continue;
                    }
                    if (tap_cols) {
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const int n = c0 + jj;
                            const int t = static_cast<int>(p.fd_cpad.div(n)), c = n - t * p.cpad;
                            if (row_ok && n < p.BN && t < I.tig && c < p.Ncols)
                                orow[c * p.os_c + p.taps[I.tap + t].btap] = __uint_as_float(r[jj]);
                        }
                        continue;
                    }
                    const int cb = I.col0 + c0;
                    if (KIND == kConv && PK != 2 && (SFV4 || UM > 1) && p.ep_vec) {
                        // lane quad = 4 consecutive q (row_ok is the same for
                        // the 4): per block of 4 columns, lane e stores column
                        // 4 b + e of the quad's 4 rows as one 16-byte run
                        const int e = lane & 3;
                        float *qrow = orow - e;
#pragma unroll
                        for (int b = 0; b < 8; ++b) {
                            uint32_t x0 = r[4 * b], x1 = r[4 * b + 1], x2 = r[4 * b + 2], x3 = r[4 * b + 3];
                            quad_transpose(x0, x1, x2, x3, e);
                            const int col = cb + 4 * b + e;
                            if (row_ok && col < p.Ncols)
                                *reinterpret_cast<float4 *>(qrow + static_cast<int64_t>(col) * p.os_c) =
                                    make_float4(__uint_as_float(x0), __uint_as_float(x1), __uint_as_float(x2),
                                                __uint_as_float(x3));
                        }
                        continue;
                    }
                    const int nv = row_ok ? min(32, p.Ncols - cb) : 0;
                    float *op = orow + static_cast<int64_t>(cb) * p.os_c;
                    if constexpr (PK == 2) {
                        const float ts = __ldg(p.nv_tx) * __ldg(p.nv_tw);   // T_x * T_w (Eq. 6 applied to both operands)
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj)
                            if (jj < nv) op[jj * p.os_c] = __uint_as_float(r[jj]) * ts;
                        continue;
                    }
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (jj < nv) op[jj * p.os_c] = __uint_as_float(r[jj]);
                }
            }
            ++tcount;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Deterministic split-K reduction: out[i] = the sum of part[s][i] over s in a
// fixed order: eight running sums (s modulo 8, each in increasing s, so
// eight loads are in flight per thread), then combined pairwise.
__global__ void splitk_reduce_kernel(const float *__restrict__ part, float *__restrict__ out, int64_t n, int splits) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float a[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
        int s = 0;
        for (; s + 8 <= splits; s += 8) {
#pragma unroll
            for (int k = 0; k < 8; ++k) a[k] += __ldg(part + (s + k) * n + i);
        }
        for (int k = 0; s < splits; ++s, ++k) a[k] += __ldg(part + s * n + i);
        out[i] = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
    }
}

// One thread waits on a barrier that nothing signals, with a time limit, so
// that the bounded wait runs out and records the device error.
__global__ void expire_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0u, limit_ns, nullptr);
    }
}

}  // namespace mqc
