// mqc.cu -- host side of libmqc: the C ABI declared in include/mqc.h.
// Validates arguments, encodes TMA tensor maps, chooses tile shapes and
// launches the kernels of quantize.cuh, im2col.cuh and conv_gemm.cuh.  It
// never allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/mqc.h"
#include "common.cuh"
#include "conv_gemm.cuh"
#include "im2col.cuh"
#include "quantize.cuh"
#include "widen.cuh"
#include "subpixel.cuh"
#include "nvfp4.cuh"

using namespace mqc;

namespace {

thread_local char g_msg[512] = "";

mqc_status fail(mqc_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return s;
}

mqc_status cuda_fail(cudaError_t e, const char *what) {
    return fail(MQC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
int64_t nb32(int64_t x) { return ceil_div(x, 32); }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool fmt_ok(int f) { return f == MQC_E4M3 || f == MQC_E5M2 || f == MQC_E2M1; }
bool mx_ok(const mqc_mx *m) {
    return m != nullptr && fmt_ok(m->fmt) && m->block >= 0 && m->block <= 2 && (m->order == 0 || m->order == 1);
}
int64_t row_elems(int fmt) { return fmt == MQC_E2M1 ? 32 : 16; }   // elements per 16-byte row unit
int emax_elem(int fmt) { return fmt == MQC_E4M3 ? 8 : (fmt == MQC_E5M2 ? 15 : 2); }

// Padded extents of the channel-batch-first layout: only the innermost axis
// is padded, to whole 16-byte rows.
void padded(int fmt, int order, int64_t A, int64_t B, int64_t &Ap, int64_t &Bp) {
    const int64_t r = row_elems(fmt);
    Ap = order == MQC_ORDER_BA ? round_up(A, r) : A;
    Bp = order == MQC_ORDER_AB ? round_up(B, r) : B;
}

int64_t codes_bytes(int fmt, int order, int64_t d0, int64_t d1, int64_t d2, int64_t d3) {
    int64_t Ap, Bp;
    padded(fmt, order, d1, d0, Ap, Bp);
    const int64_t n = d2 * d3 * Ap * Bp;
    return fmt == MQC_E2M1 ? n / 2 : n;
}

int64_t scales_bytes(int fmt, int block, int order, int64_t d0, int64_t d1, int64_t d2, int64_t d3) {
    int64_t Ap, Bp;
    padded(fmt, order, d1, d0, Ap, Bp);
    const int64_t pix = d2 * d3;
    if (block == MQC_BLOCK_A32) return pix * Bp * nb32(Ap);
    if (block == MQC_BLOCK_B32) return pix * nb32(Bp) * Ap;
    return pix * nb32(Bp) * nb32(Ap);
}

bool conv_ok(const mqc_conv *c) {
    if (c == nullptr) return false;
    if (c->N <= 0 || c->C <= 0 || c->H <= 0 || c->W <= 0 || c->K <= 0 || c->R <= 0 || c->S <= 0) return false;
    if (c->stride_h <= 0 || c->stride_w <= 0 || c->pad_h < 0 || c->pad_w < 0) return false;
    if (c->H + 2 * c->pad_h < c->R || c->W + 2 * c->pad_w < c->S) return false;
    return true;
}
int conv_P(const mqc_conv *c) { return (c->H + 2 * c->pad_h - c->R) / c->stride_h + 1; }
int conv_Q(const mqc_conv *c) { return (c->W + 2 * c->pad_w - c->S) / c->stride_w + 1; }

// ---------------------------------------------------------------- device info
struct DevInfo {
    int sms = 0;
    int max_smem = 0;
    bool gemm_attr[20] = {};  // [0] weight gradient, [1 + 3 * SFV4 + log2(um)] forward kind, [7] SFV4 weight
                              // gradient, [8 + 1 + 3 * SFV4 + log2(um)] forward with a quantized output,
                              // [8] MXFP4 and [15] NVFP4 forward on packed codes, [16 + 2 * quantized
                              // output + (um == 4)] narrow forward
    bool quant_attr[72] = {};    // staged quantizer, [36*sr + (fmt*3 + blk)*4 + tile]
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

mqc_status dev_info(DevInfo *&out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(MQC_ERR_CUDA, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo &d = g_dev[dev];
    if (d.sms == 0) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0)
            return fail(MQC_ERR_UNSUPPORTED, "libmqc is built for sm_100a; device %d is sm_%d%d", dev, major, minor);
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
        e = cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(smem)");
    }
    out = &d;
    return MQC_OK;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

mqc_status get_encoder() {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? MQC_OK : fail(MQC_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
}

// Encoded maps, reused across calls: the key is every input of the encoder
// (address, rank, extents, strides, box, swizzle), so a hit returns exactly
// what encoding would (also after a buffer is freed and another lands at the
// same address).  Direct-mapped, 256 entries, one lock.
struct MapKey {
    uint64_t base, dims[5], strides[4];
    uint32_t box[5];
    int32_t rank, wkb;
    int32_t zero;                 // keeps the key free of padding bytes (compared with memcmp)
};
static_assert(sizeof(MapKey) == 112, "MapKey must have no padding");
struct MapSlot {
    MapKey key;
    CUtensorMap map;
    bool used;
};
constexpr int kMapCacheSlots = 256;
MapSlot g_map_cache[kMapCacheSlots];
std::mutex g_map_mutex;

uint32_t map_key_hash(const MapKey &k) {
    // FNV-1a over the key's bytes
    const unsigned char *b = reinterpret_cast<const unsigned char *>(&k);
    uint32_t h = 2166136261u;
    for (size_t i = 0; i < sizeof k; ++i) h = (h ^ b[i]) * 16777619u;
    return h;
}

// Encode a tiled map over 1-byte codes.  dims[0] is contiguous; strides are
// the byte strides of dims[1..rank-1]; the inner box is 32*wkb bytes with the
// matching shared-memory swizzle.
mqc_status encode_codes_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                            const uint64_t *strides, const uint32_t *box, int wkb) {
    mqc_status st = get_encoder();
    if (st != MQC_OK) return st;
    MapKey key;
    memset(&key, 0, sizeof key);
    key.base = reinterpret_cast<uint64_t>(base);
    key.rank = rank;
    key.wkb = wkb;
    for (int i = 0; i < rank && i < 5; ++i) {
        key.dims[i] = dims[i];
        key.box[i] = box[i];
    }
    for (int i = 0; i + 1 < rank && i < 4; ++i) key.strides[i] = strides[i];
    const uint32_t slot = map_key_hash(key) % kMapCacheSlots;
    {
        std::lock_guard<std::mutex> lock(g_map_mutex);
        const MapSlot &c = g_map_cache[slot];
        if (c.used && memcmp(&c.key, &key, sizeof key) == 0) {
            *map = c.map;
            return MQC_OK;
        }
    }
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (dims[i] == 0 || dims[i] > (1ull << 32)) return fail(MQC_ERR_INVALID, "tensor extent %llu out of range",
                                                                (unsigned long long)dims[i]);
        if (box[i] == 0 || box[i] > 256) return fail(MQC_ERR_INVALID, "box extent %u out of range", box[i]);
    }
    for (int i = 0; i < rank - 1; ++i) {
        gs[i] = strides[i];
        if (strides[i] % 16 != 0) return fail(MQC_ERR_ALIGNMENT, "tensor stride %llu not a multiple of 16 bytes",
                                              (unsigned long long)strides[i]);
    }
    const CUtensorMapSwizzle sw = wkb == 4   ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : wkb == 2 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : wkb == 1 ? CU_TENSOR_MAP_SWIZZLE_32B
                                             : CU_TENSOR_MAP_SWIZZLE_NONE;   // wkb 0: plain rows
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void *>(base), gd, gs, bx, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MQC_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    if (rank <= 5) {
        std::lock_guard<std::mutex> lock(g_map_mutex);
        MapSlot &c = g_map_cache[slot];
        memcpy(&c.key, &key, sizeof key);
        c.map = *map;
        c.used = true;
    }
    return MQC_OK;
}

int largest_wkb(int64_t nblocks) { return nblocks % 4 == 0 ? 4 : (nblocks % 2 == 0 ? 2 : 1); }

// Output-tile geometry of the CONV kind: a box of bq x bp x bn output
// positions (q fastest) with at most 128 rows, chosen to minimise the rows
// computed over the whole problem, with a preference for long runs along q
// (contiguous fp32 stores in NCHW).
void choose_rows(int Qe, int Pe, int Ne, int &bq, int &bp, int &bn, int rows = 128) {
    double best = 1e300;
    bq = bp = bn = 1;
    for (int q = 1; q <= std::min(Qe, rows); ++q)
        for (int n = 1; n <= std::min(Ne, rows / q); ++n) {
            const int pr = std::min(Pe, rows / (q * n));
            if (pr < 1) continue;
            const double tiles = double(ceil_div(Qe, q)) * ceil_div(Pe, pr) * ceil_div(Ne, n);
            double cost = tiles * 128.0;
            const int want = std::min(32, Qe);
            if (q < want) cost *= 1.0 + 0.25 * (1.0 - double(q) / want);
            if (cost < best - 1e-9) {
                best = cost;
                bq = q;
                bp = pr;
                bn = n;
            }
        }
}

int choose_bn(int ncols) {
    if (ncols <= 128) return static_cast<int>(round_up(ncols, 16));
    return 128;
}

// Rows of a box that holds a whole operand tile dimension of `rows` (when it
// fits one tile): rows beyond the operand are not copied (the MMA reads stale
// shared memory there; those accumulator rows or columns are never stored).
int box_rows(int rows, int tile) { return rows < tile ? static_cast<int>(round_up(rows, 8)) : tile; }

uint32_t mma_fmt(int f) { return f == MQC_E4M3 ? 0u : (f == MQC_E5M2 ? 1u : 5u); }

const uint64_t kDefaultTimeoutNs = 4000000000ull;

FastDiv make_fastdiv(int32_t d) {
    FastDiv f;
    f.d = static_cast<uint32_t>(std::max(1, d));
    f.l = 0;
    while ((1ull << f.l) < f.d) ++f.l;
    f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << f.l) - f.d)) / f.d + 1);
    return f;
}

template <int KIND>
mqc_status launch_gemm(GemmParams &P, const DevInfo &d, cudaStream_t stream) {
    // CONV: the weights' scale atoms are the same for every output tile of a
    // column tile; build them once per CTA when they fit in 16 KB and cannot
    // be read four bytes at a time
    // groups of 4 K-blocks: per phase for CONV (their sum indexes the scale
    // cache), per unit otherwise
    if (KIND == kConv) {
        P.groups = 0;
        P.total_kb = 0;
        for (int ph = 0; ph < P.nph; ++ph) {
            P.ph_gofs[ph] = P.groups;
            P.groups += (P.ph_tkb[ph] + 3) / 4;
            P.total_kb = std::max(P.total_kb, P.ph_tkb[ph]);
        }
    } else {
        P.groups = (P.total_kb + 3) / 4;
    }
    const int pk = KIND == kConv ? P.pk : 0;                 // packed FP4 operands: 1 MXFP4, 2 NVFP4
    const bool nv = pk != 0;
    const int spk = pk == 2 ? 4 : (pk == 1 ? 2 : 1);         // scale atoms per group of 4 K-blocks
    const int cache = KIND == kConv ? P.NT * P.groups * P.nb_atoms * 512 : 0;
    P.sfb_cached = KIND == kConv && cache <= 16384 && !P.sfb_vec4 && !nv;
    // the 32-bit scale path reads B four bytes at a time unless B is cached
    // (the packed-FP4 path has its own vector loads for both operands)
    if (!P.sfb_cached && !P.sfb_vec4 && !nv) P.sf_vec4 = 0;
    // k16: the zero block (4 KB) 1 KB past the barriers; quantized output:
    // eight 32 x 36-byte transposition buffers there (after the zero block)
    const bool qout = KIND == kConv && P.q_codes != nullptr;
    // ep_stage: two 16 x 260-float buffers per epilogue team after them
    const int extra = (P.k16 || qout) ? 1024 + (P.k16 ? 4096 : 0) + (qout ? 8 * 32 * 36 : 0) +
                                            (P.ep_stage ? 2 * 2 * 16 * 260 * 4 : 0)
                                      : 64 * 8 + 64;
    const int fixed = 1024 + extra + (P.sfb_cached ? cache : 0);
    // CONV with few K-blocks per tile and narrow column tiles: units of
    // um = 2 or 4 row tiles, so that the per-unit work of every role (decode,
    // barrier round trips, B loads, scale atoms of B) is shared by um MMAs;
    // only while there are still at least two units per SM.  Measured on the
    // YOLOv8n layers: a gain up to 9 K-blocks and 32 columns, a loss with 12
    // K-blocks (the scale gather redoes the rows of every sub-tile per stage)
    // or 64 columns.
    P.um = 1;
    if (KIND == kConv) {
        P.MTILES = P.TQ * P.TP * P.TN;
        if (P.total_kb <= 9 && P.BN <= 32 && !nv) {
            for (int um = 4; um >= 2; um /= 2) {
                if (P.k16 && um == 2) continue;    // the narrow kernels come with units of 1 or 4
                const int64_t units = ceil_div(P.MTILES, um) * int64_t(P.nph) * P.NT;
                if (2 * um * P.BN <= 256 && units >= 2 * d.sms) {
                    P.um = um;
                    break;
                }
            }
        }
        P.num_units = static_cast<int32_t>(ceil_div(P.MTILES, P.um) * int64_t(P.nph) * P.NT);
    }
    auto stages_for = [&](int kbs, int &S) {
        const int ga = kbs / 4;
        const int kb_bytes = P.k16 ? 16 : 32;
        const int per_stage = P.um * 128 * kb_bytes * kbs + P.BN * kb_bytes * kbs + 512 * ga * P.um * spk +
                              512 * ga * P.nb_atoms * spk;
        const int sf_cols = ga * spk * (4 * P.um + 4 * P.nb_atoms);
        S = std::min(8, (d.max_smem - fixed) / per_stage);
        S = std::min(S, (kTmemCols - kSfTmemBase) / sf_cols);
        return per_stage;
    };
    // 8 K-blocks per stage (twice the MMAs per barrier round trip) when at
    // least 3 such stages fit and the tile has more than 4 K-blocks
    int S8 = 0, S4 = 0;
    const int ps8 = stages_for(8, S8), ps4 = stages_for(4, S4);
    const bool long_k = KIND == kConv ? P.total_kb > 4 : P.kiters_total > 1;
    P.kbs = (long_k && S8 >= 3 && P.um == 1) ? 8 : 4;
    const int S = P.kbs == 8 ? S8 : S4;
    const int per_stage = P.kbs == 8 ? ps8 : ps4;
    if (S < 3) return fail(MQC_ERR_UNSUPPORTED, "tile does not fit in shared memory");
    P.stages = S;
    P.nsf = 0;
    if (KIND == kConv && P.nph == 1) {
        // every unit has the same stages (kbs K-blocks, the last one the
        // rest): over one period of the round robin (lcm of the stages per
        // unit and the warp count), the busiest warp's K-blocks per unit,
        // each stage counted one more for its fixed cost; the fewest wins,
        // ties to more warps
        const int nk = (P.ph_tkb[0] + P.kbs - 1) / P.kbs;
        const int nmax = std::min(kNumSfWarps, S);
        double best = 1e300;
        for (int nsf = nmax; nsf >= 1 && nk > 0; --nsf) {
            int L = nk;
            while (L % nsf != 0) L += nk;
            double worst = 0.0;
            for (int w = 0; w < nsf; ++w) {
                int load = 0;
                for (int g = w; g < L; g += nsf) load += std::min(P.kbs, P.ph_tkb[0] - P.kbs * (g % nk)) + 1;
                worst = std::max(worst, double(load) * nk / L);
            }
            if (worst < best - 1e-9) {
                best = worst;
                P.nsf = nsf;
            }
        }
    }
    if (P.sub < 1) P.sub = 1;
    P.fd_NT = make_fastdiv(P.NT);
    P.fd_nph = make_fastdiv(P.nph);
    P.fd_TQ = make_fastdiv(P.TQ);
    P.fd_TP = make_fastdiv(P.TP);
    P.fd_sub = make_fastdiv(P.sub);
    P.fd_bq = make_fastdiv(P.bq);
    P.fd_bp = make_fastdiv(P.bp);
    P.fd_bn = make_fastdiv(P.bn);
    P.fd_MT = make_fastdiv(P.MT);
    P.fd_ngroups = make_fastdiv(P.ngroups);
    P.fd_cpad = make_fastdiv(P.cpad);
    P.fd_splits = make_fastdiv(P.splits);
    if (KIND == kWgrad && int64_t(P.kiters_total) * (P.splits + 1) >= (1ll << 31))
        return fail(MQC_ERR_UNSUPPORTED, "weight gradient: reduction too long");
    // accumulators in TMEM columns [0, 256): as many as fit, up to 4, so that
    // several tiles can wait between the MMA issuer and the epilogue
    const int acc_cols = P.um * P.BN;   // TMEM columns of one unit's accumulators
    P.nacc = acc_cols <= 64 ? 4 : (acc_cols <= 128 ? 2 : 1);
    P.lg_nacc = P.nacc == 4 ? 2 : (P.nacc == 2 ? 1 : 0);
    P.timeout_ns = kDefaultTimeoutNs;
    const int smem = fixed + S * per_stage;
    const bool v4 = KIND == kConv && P.sf_vec4;
    auto kernel = P.sq_gather ? conv_gemm_kernel<kWgrad, true, 1> : conv_gemm_kernel<kWgrad, false, 1>;
    if (KIND == kConv && P.k16) {
        if (qout) kernel = P.um == 4 ? conv_gemm_kernel<kConv, false, 4, true, 0, true> : conv_gemm_kernel<kConv, false, 1, true, 0, true>;
        else kernel = P.um == 4 ? conv_gemm_kernel<kConv, false, 4, false, 0, true> : conv_gemm_kernel<kConv, false, 1, false, 0, true>;
    } else if (pk == 2) {
        kernel = conv_gemm_kernel<kConv, false, 1, false, 2>;
    } else if (pk == 1) {
        kernel = conv_gemm_kernel<kConv, false, 1, false, 1>;
    } else if (KIND == kConv && !qout) {
        if (P.um == 4) kernel = v4 ? conv_gemm_kernel<kConv, true, 4> : conv_gemm_kernel<kConv, false, 4>;
        else if (P.um == 2) kernel = v4 ? conv_gemm_kernel<kConv, true, 2> : conv_gemm_kernel<kConv, false, 2>;
        else kernel = v4 ? conv_gemm_kernel<kConv, true, 1> : conv_gemm_kernel<kConv, false, 1>;
    } else if (KIND == kConv) {
        if (P.um == 4) kernel = v4 ? conv_gemm_kernel<kConv, true, 4, true> : conv_gemm_kernel<kConv, false, 4, true>;
        else if (P.um == 2) kernel = v4 ? conv_gemm_kernel<kConv, true, 2, true> : conv_gemm_kernel<kConv, false, 2, true>;
        else kernel = v4 ? conv_gemm_kernel<kConv, true, 1, true> : conv_gemm_kernel<kConv, false, 1, true>;
    }
    const int ai = KIND == kConv && P.k16 ? 16 + (qout ? 2 : 0) + (P.um == 4 ? 1 : 0)
                   : pk == 2 ? 15 : pk == 1 ? 8
                      : KIND == kConv ? (qout ? 8 : 0) + 1 + (v4 ? 3 : 0) + (P.um == 4 ? 2 : P.um - 1)
                                      : (P.sq_gather ? 7 : 0);
    if (!d.gemm_attr[ai]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, d.max_smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        const_cast<DevInfo &>(d).gemm_attr[ai] = true;
    }
    // vector stores of the plain fp32 epilogue: rows q-consecutive in lane
    // quads (no slots, q fastest, whole quads per p row), every row start and
    // stride a multiple of 4 floats, the output 16-byte aligned
    P.ep_vec = 0;
    if (KIND == kConv && !P.k16 && !qout && pk == 0 && (P.sf_vec4 || P.um > 1) && P.d2s == 0 && P.sub == 1 &&
        !P.rows_nfirst && P.bq % 4 == 0 &&
        P.os_q == 1 && P.os_p % 4 == 0 && P.os_c % 4 == 0 && P.os_n % 4 == 0 &&
        (reinterpret_cast<uintptr_t>(P.out) & 15u) == 0) {
        bool ok4 = true;
        for (int ph = 0; ph < P.nph; ++ph) ok4 = ok4 && P.ph_out_base[ph] % 4 == 0 && P.ph_Qe[ph] % 4 == 0;
        P.ep_vec = ok4 ? 1 : 0;
    }
    const int grid = std::max(1, std::min(P.num_units, d.sms));
    kernel<<<grid, gemm_threads<KIND>(), smem, stream>>>(P);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "conv_gemm_kernel launch");
    return MQC_OK;
}

// Tap of a strided operand: r - pad = st*d + phase with 0 <= phase < st.
void split_tap(int off, int st, int &d, int &ph) {
    ph = ((off % st) + st) % st;
    d = (off - ph) / st;
}

bool gemm_fmt_ok(const mqc_mx *m) { return m->fmt == MQC_E4M3 || m->fmt == MQC_E5M2 || m->fmt == MQC_E2M1; }

// A GEMM operand as the kernel reads it: FP8 codes as given; E2M1 codes
// rewritten as the E4M3 codes of the same values into the workspace (same
// layout, one byte per element), so the tensor core runs every format
// through kind::mxf8f6f4 with unchanged E8M0 scales.
struct GemmOperand {
    const uint8_t *codes;
    int mma_fmt;       // element format the MMA reads (E4M3 or E5M2)
    int64_t inner;     // padded innermost extent: elements = bytes of one row
};

// Workspace bytes of the widened copy of an operand [d0=B][d1=A][d2][d3].
size_t widened_bytes(const mqc_mx *m, int64_t d0, int64_t d1, int64_t d2, int64_t d3) {
    if (m->fmt != MQC_E2M1) return 0;
    return static_cast<size_t>(round_up(2 * codes_bytes(MQC_E2M1, m->order, d0, d1, d2, d3), 256));
}

mqc_status check_workspace(const char *name, const void *ws, size_t bytes, size_t need) {
    if (need == 0) return MQC_OK;
    if (ws == nullptr || bytes < need) return fail(MQC_ERR_WORKSPACE, "%s: needs %zu workspace bytes", name, need);
    if (!aligned16(ws)) return fail(MQC_ERR_ALIGNMENT, "%s: workspace not 16-byte aligned", name);
    return MQC_OK;
}

// Fills o for the operand [d0][d1][d2][d3] with codes q; an E2M1 operand is
// widened into *wsp, which then advances past the copy.
mqc_status gemm_operand(const void *q, const mqc_mx *m, int64_t d0, int64_t d1, int64_t d2, int64_t d3, uint8_t *&wsp,
                        cudaStream_t s, GemmOperand &o) {
    int64_t Ap, Bp;
    padded(m->fmt, m->order, d1, d0, Ap, Bp);
    o.inner = m->order == MQC_ORDER_BA ? Ap : Bp;
    if (m->fmt != MQC_E2M1) {
        o.codes = static_cast<const uint8_t *>(q);
        o.mma_fmt = m->fmt;
        return MQC_OK;
    }
    const int64_t nb = codes_bytes(MQC_E2M1, m->order, d0, d1, d2, d3);   // a multiple of 16 (16-byte rows)
    const int64_t chunks = nb / 16;
    if (chunks > 0) {
        const int blocks = static_cast<int>(std::min<int64_t>(ceil_div(chunks, 256), 148 * 16));
        widen_e2m1_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint8_t *>(q), wsp, chunks);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "widen_e2m1_kernel launch");
    }
    o.codes = wsp;
    o.mma_fmt = MQC_E4M3;
    wsp += widened_bytes(m, d0, d1, d2, d3);
    return MQC_OK;
}

mqc_status check_gemm_operand(const char *name, const void *q, const uint8_t *s, const mqc_mx *m, int want_order,
                              bool along_first) {
    if (q == nullptr || s == nullptr || !mx_ok(m)) return fail(MQC_ERR_INVALID, "%s: null pointer or bad mx", name);
    if (!aligned16(q)) return fail(MQC_ERR_ALIGNMENT, "%s codes not 16-byte aligned", name);
    if (!gemm_fmt_ok(m)) return fail(MQC_ERR_UNSUPPORTED, "%s: unknown element format", name);
    if (m->order != want_order)
        return fail(MQC_ERR_UNSUPPORTED, "%s: code order must be %s", name, want_order == 0 ? "BA" : "AB");
    const int want_block = along_first ? MQC_BLOCK_A32 : MQC_BLOCK_B32;
    if (m->block != want_block && m->block != MQC_BLOCK_SQ32)
        return fail(MQC_ERR_UNSUPPORTED, "%s: block mode must be %s or SQ32", name, along_first ? "A32" : "B32");
    return MQC_OK;
}

}  // namespace

extern "C" {

int32_t mqc_version(void) { return 100; }

const char *mqc_status_string(mqc_status s) {
    switch (s) {
    case MQC_OK: return "ok";
    case MQC_ERR_INVALID: return "invalid argument";
    case MQC_ERR_UNSUPPORTED: return "unsupported";
    case MQC_ERR_CUDA: return "CUDA error";
    case MQC_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case MQC_ERR_ALIGNMENT: return "misaligned pointer";
    case MQC_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

const char *mqc_last_error_message(void) { return g_msg; }

int64_t mqc_codes_bytes(const mqc_mx *mx, int32_t d0, int32_t d1, int32_t d2, int32_t d3) {
    if (!mx_ok(mx) || d0 <= 0 || d1 <= 0 || d2 <= 0 || d3 <= 0) return -1;
    return codes_bytes(mx->fmt, mx->order, d0, d1, d2, d3);
}

int64_t mqc_scales_bytes(const mqc_mx *mx, int32_t d0, int32_t d1, int32_t d2, int32_t d3) {
    if (!mx_ok(mx) || d0 <= 0 || d1 <= 0 || d2 <= 0 || d3 <= 0) return -1;
    return scales_bytes(mx->fmt, mx->block, mx->order, d0, d1, d2, d3);
}

mqc_status mqc_tensor_dims(mqc_role role, const mqc_conv *c, int32_t dims[4]) {
    if (!conv_ok(c) || dims == nullptr) return fail(MQC_ERR_INVALID, "bad conv descriptor");
    switch (role) {
    case MQC_ROLE_X: dims[0] = c->N; dims[1] = c->C; dims[2] = c->H; dims[3] = c->W; return MQC_OK;
    case MQC_ROLE_W: dims[0] = c->K; dims[1] = c->C; dims[2] = c->R; dims[3] = c->S; return MQC_OK;
    case MQC_ROLE_G: dims[0] = c->N; dims[1] = c->K; dims[2] = conv_P(c); dims[3] = conv_Q(c); return MQC_OK;
    }
    return fail(MQC_ERR_INVALID, "bad role %d", (int)role);
}

}  // extern "C"

// ------------------------------------------------------------------ quantize
// Stochastic rounding request: Philox key and stream offset.
struct SrArgs {
    uint64_t seed, offset;
};

static mqc_status quantize_impl(const float *src, const mqc_t4 *d, const mqc_mx *mx, void *codes, uint8_t *scales,
                                void *codes_alt, void *stream, const SrArgs *sr);

extern "C" {

mqc_status mqc_quantize_mx(const float *src, const mqc_t4 *d, const mqc_mx *mx, void *codes, uint8_t *scales,
                           void *codes_alt, void *stream) {
    return quantize_impl(src, d, mx, codes, scales, codes_alt, stream, nullptr);
}

mqc_status mqc_quantize_mx_sr(const float *src, const mqc_t4 *d, const mqc_mx *mx, void *codes, uint8_t *scales,
                              void *codes_alt, uint64_t seed, uint64_t offset, void *stream) {
    const SrArgs sr{seed, offset};
    return quantize_impl(src, d, mx, codes, scales, codes_alt, stream, &sr);
}

}  // extern "C"

// Argument checks shared by the quantization entry points.
static mqc_status check_quant_args(const float *src, const mqc_t4 *d, const mqc_mx *mx, const void *codes,
                                   const uint8_t *scales, const void *codes_alt) {
    if (src == nullptr || d == nullptr || codes == nullptr || scales == nullptr || !mx_ok(mx))
        return fail(MQC_ERR_INVALID, "quantize: null pointer or bad mx descriptor");
    if (d->d0 <= 0 || d->d1 <= 0 || d->d2 <= 0 || d->d3 <= 0)
        return fail(MQC_ERR_INVALID, "quantize: extents must be positive");
    if ((reinterpret_cast<uintptr_t>(src) & 3u) != 0) return fail(MQC_ERR_ALIGNMENT, "quantize: src not 4-byte aligned");
    if (!aligned16(codes) || (codes_alt != nullptr && !aligned16(codes_alt)))
        return fail(MQC_ERR_ALIGNMENT, "quantize: codes not 16-byte aligned");
    if (static_cast<int64_t>(d->d2) * d->d3 > (int64_t(1) << 31) - 64)
        return fail(MQC_ERR_INVALID, "quantize: too many spatial positions");
    return MQC_OK;
}

// Parameters and tile count of the generic quantizer (mx_quantize_kernel)
// for one tensor; `it` = 16 or 32 codes per tile row (0: choose).
static void generic_quant_params(const float *src, const mqc_t4 *d, const mqc_mx *mx, void *codes, uint8_t *scales,
                                 void *codes_alt, int it_req, QuantParams &p, int &it, int64_t &tiles) {
    p = QuantParams{};
    p.src = src;
    p.sb = d->s0;
    p.sa = d->s1;
    p.sh = d->s2;
    p.sw = d->s3;
    p.B = d->d0;
    p.A = d->d1;
    p.H = d->d2;
    p.W = d->d3;
    p.npix = d->d2 * d->d3;
    int64_t Ap, Bp;
    padded(mx->fmt, mx->order, p.A, p.B, Ap, Bp);
    p.Ap1 = static_cast<int32_t>(Ap);
    p.Bp1 = static_cast<int32_t>(Bp);
    const bool map_a = mx->order == MQC_ORDER_BA;
    const bool fp4 = mx->fmt == MQC_E2M1;
    const int64_t r = row_elems(mx->fmt);
    p.I = map_a ? p.A : p.B;
    p.O = map_a ? p.B : p.A;
    p.I1 = static_cast<int32_t>(map_a ? Ap : Bp);
    p.codes = static_cast<uint8_t *>(codes);
    p.codes_alt = static_cast<uint8_t *>(codes_alt);
    p.O2 = static_cast<int32_t>(round_up(p.O, r));
    p.scales = scales;
    p.fmt = mx->fmt;
    p.emax = emax_elem(mx->fmt);
    // tile: IT = 16 when the innermost axis holds at most 16 FP8 codes, OT = 16
    // when the other axis (and its padded copy) has at most 16 elements
    it = it_req ? it_req : ((!fp4 && p.I1 <= 16) ? 16 : 32);
    p.OT = (!fp4 && p.O <= 16 && (codes_alt == nullptr || p.O2 <= 16)) ? 16 : 32;
    const int gsize = p.OT == 16 ? 2 : 1;
    p.nPT = static_cast<int32_t>(ceil_div(p.npix, 32 * gsize));
    p.nIT = static_cast<int32_t>(ceil_div(p.I1, it));
    p.nOT = static_cast<int32_t>(ceil_div(codes_alt ? std::max(p.O, p.O2) : p.O, p.OT));
    tiles = int64_t(p.nPT) * p.nOT * p.nIT;
}

static mqc_status quantize_impl(const float *src, const mqc_t4 *d, const mqc_mx *mx, void *codes, uint8_t *scales,
                                void *codes_alt, void *stream, const SrArgs *sr) {
    mqc_status st = check_quant_args(src, d, mx, codes, scales, codes_alt);
    if (st != MQC_OK) return st;
    // staged kernel: positions contiguous (element stride 1 along W, W along
    // H), every plane 16-byte aligned
    const bool staged = d->s3 == 1 && d->s2 == d->d3 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
                        d->s0 % 4 == 0 && d->s1 % 4 == 0;
    if (sr != nullptr && (mx->order != MQC_ORDER_BA || !staged))
        return fail(MQC_ERR_UNSUPPORTED,
                    "quantize_mx_sr: needs order BA and an NCHW-like source (contiguous, 16-byte aligned planes)");
    DevInfo *dv;
    if ((st = dev_info(dv)) != MQC_OK) return st;

    QuantParams p;
    int it;
    int64_t tiles;
    generic_quant_params(src, d, mx, codes, scales, codes_alt, 0, p, it, tiles);
    if (tiles > (int64_t(1) << 31) - 1) return fail(MQC_ERR_INVALID, "quantize: tensor too large");
    const bool map_a = mx->order == MQC_ORDER_BA;
    const bool fp4 = mx->fmt == MQC_E2M1;
    const bool along_i = (mx->block == MQC_BLOCK_A32) == map_a && mx->block != MQC_BLOCK_SQ32;
    const int blk = mx->block == MQC_BLOCK_SQ32 ? kSquare : (along_i ? kAlongI : kAlongO);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool dual = codes_alt != nullptr;
    if (staged) {
        StagedParams sp{};
        sp.q = p;
        sp.IT = (!fp4 && p.I1 <= 16) ? 16 : 32;     // FP4 rows are 32 codes
        sp.OT = (dual ? std::max(p.O, p.O2) : p.O) <= 16 ? 16 : 32;
        sp.PT = kStagedTileBytes / (4 * sp.OT * sp.IT);
        sp.nPT = static_cast<int32_t>(ceil_div(p.npix, sp.PT));
        sp.nOT = static_cast<int32_t>(ceil_div(dual ? std::max(p.O, p.O2) : p.O, sp.OT));
        sp.nIT = static_cast<int32_t>(ceil_div(p.I1, sp.IT));
        sp.blk = blk;
        sp.map_a = map_a ? 1 : 0;
        if (sr != nullptr) {
            sp.seed = sr->seed;
            sp.offset = sr->offset;
            sp.a16_blocks = static_cast<int32_t>(ceil_div(p.A, 16));
        }
        const int64_t ntiles = int64_t(sp.nPT) * sp.nOT * sp.nIT;
        if (ntiles > (int64_t(1) << 31) - 1) return fail(MQC_ERR_INVALID, "quantize: tensor too large");
        // tile, block reciprocals, square maxima (+ the codes of the tile with SR)
        const int smem = kStagedTileBytes + 32 * 64 * 4 + 64 * 4 + (sr ? kStagedTileBytes / 4 : 0);
        // the shared-memory limit is raised once per (SR, format, block, tile) kernel
        const int ai = (sr ? 36 : 0) + (p.fmt * 3 + blk) * 4 + (sp.OT == 32 ? 2 : 0) + (sp.IT == 32 ? 1 : 0);
        cudaError_t ae = cudaSuccess;
        const unsigned g = static_cast<unsigned>(ntiles);
        const bool set = !dv->quant_attr[ai];
        if (sr == nullptr) {
            if (p.fmt == MQC_E4M3) launch_staged<0, false>(sp, g, smem, s, ae, set);
            else if (p.fmt == MQC_E5M2) launch_staged<1, false>(sp, g, smem, s, ae, set);
            else launch_staged<2, false>(sp, g, smem, s, ae, set);
        } else {
            if (p.fmt == MQC_E4M3) launch_staged<0, true>(sp, g, smem, s, ae, set);
            else if (p.fmt == MQC_E5M2) launch_staged<1, true>(sp, g, smem, s, ae, set);
            else launch_staged<2, true>(sp, g, smem, s, ae, set);
        }
        if (ae != cudaSuccess) return cuda_fail(ae, "cudaFuncSetAttribute");
        dv->quant_attr[ai] = true;
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "mx_quantize_staged_kernel launch");
        return MQC_OK;
    }
    if (map_a) launch_quantize_blk<true>(p, blk, dual, it, static_cast<unsigned>(tiles), s);
    else launch_quantize_blk<false>(p, blk, dual, it, static_cast<unsigned>(tiles), s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "mx_quantize_kernel launch");
    return MQC_OK;
}

extern "C" {

int64_t mqc_nvfp4_scales_bytes(int32_t block, int32_t order, int32_t d0, int32_t d1, int32_t d2, int32_t d3) {
    if (block < 0 || block > 2 || (order != 0 && order != 1) || d0 <= 0 || d1 <= 0 || d2 <= 0 || d3 <= 0) return -1;
    int64_t Ap, Bp;
    padded(MQC_E2M1, order, d1, d0, Ap, Bp);
    const int64_t pix = int64_t(d2) * d3;
    if (block == MQC_NV_A16) return pix * Bp * ceil_div(Ap, 16);
    if (block == MQC_NV_B16) return pix * ceil_div(Bp, 16) * Ap;
    return pix * ceil_div(Bp, 16) * ceil_div(Ap, 16);
}

mqc_status mqc_quantize_nvfp4(const float *src, const mqc_t4 *d, int32_t block, int32_t order, void *codes,
                              uint8_t *scales, void *codes_alt, float *tscale, void *stream) {
    if (src == nullptr || d == nullptr || codes == nullptr || scales == nullptr || tscale == nullptr ||
        block < 0 || block > 2 || (order != 0 && order != 1))
        return fail(MQC_ERR_INVALID, "quantize_nvfp4: null pointer or bad block / order");
    if (d->d0 <= 0 || d->d1 <= 0 || d->d2 <= 0 || d->d3 <= 0)
        return fail(MQC_ERR_INVALID, "quantize_nvfp4: extents must be positive");
    if ((reinterpret_cast<uintptr_t>(src) & 3u) != 0 || (reinterpret_cast<uintptr_t>(tscale) & 3u) != 0)
        return fail(MQC_ERR_ALIGNMENT, "quantize_nvfp4: src / tscale not 4-byte aligned");
    if (!aligned16(codes) || (codes_alt != nullptr && !aligned16(codes_alt)))
        return fail(MQC_ERR_ALIGNMENT, "quantize_nvfp4: codes not 16-byte aligned");
    if (d->s3 != 1 || d->s2 != d->d3)
        return fail(MQC_ERR_UNSUPPORTED, "quantize_nvfp4: spatial positions must be contiguous (NCHW-like)");
    if (int64_t(d->d2) * d->d3 > (int64_t(1) << 31) - 64)
        return fail(MQC_ERR_INVALID, "quantize_nvfp4: too many spatial positions");
    DevInfo *dv;
    mqc_status st = dev_info(dv);
    if (st != MQC_OK) return st;
    NvParams p{};
    p.src = src;
    p.sb = d->s0;
    p.sa = d->s1;
    p.B = d->d0;
    p.A = d->d1;
    p.npix = d->d2 * d->d3;
    int64_t Ap, Bp, Ap2, Bp2;
    padded(MQC_E2M1, order, p.A, p.B, Ap, Bp);
    padded(MQC_E2M1, 1 - order, p.A, p.B, Ap2, Bp2);
    p.Ap = static_cast<int32_t>(Ap);
    p.Bp = static_cast<int32_t>(Bp);
    p.Ap_alt = static_cast<int32_t>(Ap2);
    p.Bp_alt = static_cast<int32_t>(Bp2);
    p.order = order;
    p.block = block;
    const int64_t Acov = codes_alt ? std::max(Ap, Ap2) : Ap, Bcov = codes_alt ? std::max(Bp, Bp2) : Bp;
    p.ntb = static_cast<int32_t>(ceil_div(Bcov, 16));
    p.nta = static_cast<int32_t>(ceil_div(Acov, 16));
    p.codes = static_cast<uint8_t *>(codes);
    p.codes_alt = static_cast<uint8_t *>(codes_alt);
    p.scales = scales;
    p.tscale = tscale;
    const int64_t ntiles = int64_t(p.npix) * p.ntb * p.nta;
    if (ntiles > (int64_t(1) << 40)) return fail(MQC_ERR_INVALID, "quantize_nvfp4: tensor too large");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(tscale + 1, 0, sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(max|X|)");
    const int64_t total = int64_t(p.B) * p.A * p.npix;
    const int ga = static_cast<int>(std::min<int64_t>(ceil_div(total, 256), int64_t(dv->sms) * 8));
    nv_amax_kernel<<<std::max(1, ga), 256, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "nv_amax_kernel launch");
    nv_quantize_kernel<<<static_cast<unsigned>(ceil_div(ntiles, 128)), 128, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "nv_quantize_kernel launch");
    return MQC_OK;
}

mqc_status mqc_quantize_mx_batch(int32_t count, const float *const *srcs, const mqc_t4 *descs, const mqc_mx *mx,
                                 void *const *codes, uint8_t *const *scales, void *const *codes_alt, void *stream) {
    if (count < 1 || count > kMaxQuantBatch || srcs == nullptr || descs == nullptr || codes == nullptr ||
        scales == nullptr || !mx_ok(mx))
        return fail(MQC_ERR_INVALID, "quantize_mx_batch: count must be 1..%d, with non-null arrays", kMaxQuantBatch);
    const bool dual = codes_alt != nullptr;
    QuantBatch b{};
    b.n = count;
    int64_t total = 0;
    for (int i = 0; i < count; ++i) {
        void *alt = dual ? codes_alt[i] : nullptr;
        if (dual && alt == nullptr)
            return fail(MQC_ERR_INVALID, "quantize_mx_batch: codes_alt[%d] is null (all or none)", i);
        mqc_status st = check_quant_args(srcs[i], &descs[i], mx, codes[i], scales[i], alt);
        if (st != MQC_OK) return st;
        int it;
        int64_t tiles;
        generic_quant_params(srcs[i], &descs[i], mx, codes[i], scales[i], alt, 32, b.q[i], it, tiles);
        b.tile0[i] = static_cast<int32_t>(total);
        total += tiles;
        if (total > (int64_t(1) << 31) - 1) return fail(MQC_ERR_INVALID, "quantize_mx_batch: tensors too large");
    }
    b.tile0[count] = static_cast<int32_t>(total);
    DevInfo *dv;
    mqc_status st = dev_info(dv);
    if (st != MQC_OK) return st;
    const bool map_a = mx->order == MQC_ORDER_BA;
    const bool along_i = (mx->block == MQC_BLOCK_A32) == map_a && mx->block != MQC_BLOCK_SQ32;
    const int blk = mx->block == MQC_BLOCK_SQ32 ? kSquare : (along_i ? kAlongI : kAlongO);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (map_a) launch_quantize_batch<true>(b, blk, mx->fmt, dual, static_cast<unsigned>(total), s);
    else launch_quantize_batch<false>(b, blk, mx->fmt, dual, static_cast<unsigned>(total), s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "mx_quantize_batch_kernel launch");
    return MQC_OK;
}

}  // extern "C"

extern "C" {

// ------------------------------------------------------------------ im2col
static void im2col_geometry(const mqc_conv *c, const mqc_mx *mx, int64_t &Ap, int64_t &Bp, int64_t &chunk_codes,
                            int64_t &rows_codes, int64_t &chunk_sc, int64_t &rows_sc) {
    padded(mx->fmt, mx->order, c->C, c->N, Ap, Bp);
    const int64_t bytes_per = mx->fmt == MQC_E2M1 ? 2 : 1;   // elements per byte
    if (mx->order == MQC_ORDER_BA) {
        chunk_codes = Ap / bytes_per;
        rows_codes = Bp;
    } else {
        chunk_codes = Ap * Bp / bytes_per;
        rows_codes = 1;
    }
    if (mx->block == MQC_BLOCK_A32) {
        rows_sc = Bp;
        chunk_sc = nb32(Ap);
    } else if (mx->block == MQC_BLOCK_B32) {
        rows_sc = nb32(Bp);
        chunk_sc = Ap;
    } else {
        rows_sc = nb32(Bp);
        chunk_sc = nb32(Ap);
    }
}

int64_t mqc_im2col_cbf_codes_bytes(const mqc_conv *c, const mqc_mx *mx) {
    if (!conv_ok(c) || !mx_ok(mx)) return -1;
    int64_t Ap, Bp, cc, rc, cs, rs;
    im2col_geometry(c, mx, Ap, Bp, cc, rc, cs, rs);
    return int64_t(conv_P(c)) * conv_Q(c) * rc * c->R * c->S * cc;
}

int64_t mqc_im2col_cbf_scales_bytes(const mqc_conv *c, const mqc_mx *mx) {
    if (!conv_ok(c) || !mx_ok(mx)) return -1;
    int64_t Ap, Bp, cc, rc, cs, rs;
    im2col_geometry(c, mx, Ap, Bp, cc, rc, cs, rs);
    return int64_t(conv_P(c)) * conv_Q(c) * rs * c->R * c->S * cs;
}

mqc_status mqc_im2col_cbf(const void *codes, const uint8_t *scales, const mqc_conv *c, const mqc_mx *mx,
                          void *codes_out, uint8_t *scales_out, void *stream) {
    if (codes == nullptr || scales == nullptr || codes_out == nullptr || scales_out == nullptr || !conv_ok(c) ||
        !mx_ok(mx))
        return fail(MQC_ERR_INVALID, "im2col: null pointer or bad descriptor");
    if (!aligned16(codes) || !aligned16(codes_out)) return fail(MQC_ERR_ALIGNMENT, "im2col: codes not 16-byte aligned");
    DevInfo *dv;
    mqc_status st = dev_info(dv);
    if (st != MQC_OK) return st;
    int64_t Ap, Bp, cc, rc, cs, rs;
    im2col_geometry(c, mx, Ap, Bp, cc, rc, cs, rs);
    Im2colParams p{};
    p.RS = c->R * c->S;
    p.S = c->S;
    p.P = conv_P(c);
    p.Q = conv_Q(c);
    p.H = c->H;
    p.W = c->W;
    p.st_h = c->stride_h;
    p.st_w = c->stride_w;
    p.pad_h = c->pad_h;
    p.pad_w = c->pad_w;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int blocks = dv->sms * 8;
    p.src = static_cast<const uint8_t *>(codes);
    p.dst = static_cast<uint8_t *>(codes_out);
    p.chunk = cc;
    p.per_pix = rc;
    p.n_out = int64_t(p.P) * p.Q * rc * p.RS * cc / 16;
    im2col_gather_kernel<true><<<blocks, 256, 0, s>>>(p);
    p.src = scales;
    p.dst = scales_out;
    p.chunk = cs;
    p.per_pix = rs;
    p.n_out = int64_t(p.P) * p.Q * rs * p.RS * cs;
    im2col_gather_kernel<false><<<blocks, 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "im2col_gather_kernel launch");
    return MQC_OK;
}

// ------------------------------------------------------------------ forward
size_t mqc_conv2d_fwd_workspace_bytes(const mqc_conv *c, const mqc_mx *xf, const mqc_mx *wf) {
    if (!conv_ok(c) || !mx_ok(xf) || !mx_ok(wf)) return 0;
    return widened_bytes(xf, c->N, c->C, c->H, c->W) + widened_bytes(wf, c->K, c->C, c->R, c->S);
}

}  // extern "C"

// Quantized output of the forward (the next layer's input, quantized in the
// GEMM epilogue): format, block mode, activation and destination buffers.
struct QoutArgs {
    const mqc_mx *yf;
    int act;
    void *yq, *yq_alt;
    uint8_t *ys;
    float *y;      // optional fp32 copy of the activated output
};

// NVFP4 operands of the forward: per-tensor scales and block modes.
struct NvArgs {
    const float *x_tscale, *w_tscale;
    int x_block, w_block;
};

static mqc_status conv_fwd_impl(const void *xq, const uint8_t *xs, const mqc_mx *xf, const void *wq,
                                const uint8_t *ws, const mqc_mx *wf, const mqc_conv *c, float *y, void *workspace,
                                size_t workspace_bytes, void *stream, const QoutArgs *qo, const NvArgs *nva = nullptr);

extern "C" {

mqc_status mqc_conv2d_fwd(const void *xq, const uint8_t *xs, const mqc_mx *xf, const void *wq, const uint8_t *ws,
                          const mqc_mx *wf, const mqc_conv *c, float *y, void *workspace, size_t workspace_bytes,
                          void *stream) {
    if (!conv_ok(c) || y == nullptr) return fail(MQC_ERR_INVALID, "conv2d_fwd: bad conv descriptor or null output");
    return conv_fwd_impl(xq, xs, xf, wq, ws, wf, c, y, workspace, workspace_bytes, stream, nullptr);
}

mqc_status mqc_conv2d_fwd_quant(const void *xq, const uint8_t *xs, const mqc_mx *xf, const void *wq,
                                const uint8_t *ws, const mqc_mx *wf, const mqc_conv *c, int32_t act,
                                const mqc_mx *yf, void *yq, uint8_t *ys, void *yq_alt, float *y, void *workspace,
                                size_t workspace_bytes, void *stream) {
    if (!conv_ok(c) || yq == nullptr || ys == nullptr || !mx_ok(yf))
        return fail(MQC_ERR_INVALID, "conv2d_fwd_quant: bad conv descriptor, output or output format");
    if (act < MQC_ACT_NONE || act > MQC_ACT_SILU) return fail(MQC_ERR_INVALID, "conv2d_fwd_quant: bad activation");
    if (yf->order != MQC_ORDER_BA || yf->block == MQC_BLOCK_B32)
        return fail(MQC_ERR_UNSUPPORTED, "conv2d_fwd_quant: the output is written in order BA, blocks A32 or SQ32");
    if (!aligned16(yq) || (yq_alt != nullptr && !aligned16(yq_alt)))
        return fail(MQC_ERR_ALIGNMENT, "conv2d_fwd_quant: output codes not 16-byte aligned");
    if (y != nullptr && (reinterpret_cast<uintptr_t>(y) & 3u) != 0)
        return fail(MQC_ERR_ALIGNMENT, "conv2d_fwd_quant: fp32 output not 4-byte aligned");
    const QoutArgs qo{yf, act, yq, yq_alt, ys, y};
    return conv_fwd_impl(xq, xs, xf, wq, ws, wf, c, y, workspace, workspace_bytes, stream, &qo);
}

mqc_status mqc_conv2d_fwd_nvfp4(const void *xq, const uint8_t *xs, const float *x_tscale, int32_t x_block,
                                const void *wq, const uint8_t *ws, const float *w_tscale, int32_t w_block,
                                const mqc_conv *c, float *y, void *stream) {
    if (!conv_ok(c) || y == nullptr || xq == nullptr || xs == nullptr || wq == nullptr || ws == nullptr ||
        x_tscale == nullptr || w_tscale == nullptr)
        return fail(MQC_ERR_INVALID, "conv2d_fwd_nvfp4: bad conv descriptor or null pointer");
    if ((x_block != MQC_NV_A16 && x_block != MQC_NV_SQ16) || (w_block != MQC_NV_A16 && w_block != MQC_NV_SQ16))
        return fail(MQC_ERR_UNSUPPORTED, "conv2d_fwd_nvfp4: operands need blocks along C (A16 or SQ16), order BA");
    if (!aligned16(xq) || !aligned16(wq)) return fail(MQC_ERR_ALIGNMENT, "conv2d_fwd_nvfp4: codes not 16-byte aligned");
    const NvArgs nva{x_tscale, w_tscale, x_block, w_block};
    const mqc_mx fx{MQC_E2M1, MQC_BLOCK_A32, MQC_ORDER_BA};   // the code layout of E2M1 (the blocks are nva's)
    return conv_fwd_impl(xq, xs, &fx, wq, ws, &fx, c, y, nullptr, 0, stream, nullptr, &nva);
}

}  // extern "C"

static mqc_status conv_fwd_impl(const void *xq, const uint8_t *xs, const mqc_mx *xf, const void *wq,
                                const uint8_t *ws, const mqc_mx *wf, const mqc_conv *c, float *y, void *workspace,
                                size_t workspace_bytes, void *stream, const QoutArgs *qo, const NvArgs *nva) {
    mqc_status st = check_gemm_operand("X", xq, xs, xf, MQC_ORDER_BA, true);
    if (st != MQC_OK) return st;
    st = check_gemm_operand("W", wq, ws, wf, MQC_ORDER_BA, true);
    if (st != MQC_OK) return st;
    if (c->R * c->S > kMaxTaps) return fail(MQC_ERR_UNSUPPORTED, "conv2d_fwd: at most %d kernel taps", kMaxTaps);
    // one activation tensor map per stride phase, four at most
    if (c->stride_h * c->stride_w > 4) return fail(MQC_ERR_UNSUPPORTED, "conv2d_fwd: stride product above 4");
    DevInfo *dv;
    if ((st = dev_info(dv)) != MQC_OK) return st;

    const int N = c->N, C = c->C, H = c->H, W = c->W, K = c->K, R = c->R, S = c->S;
    const int sh = c->stride_h, sw = c->stride_w, P = conv_P(c), Q = conv_Q(c);
    GemmOperand ox, ow;
    // both operands OCP MXFP4 (plain forward): the packed codes go to the
    // tensor core as they are (kind::mxf4), no widening
    const bool mxf4 = nva == nullptr && qo == nullptr && xf->fmt == MQC_E2M1 && wf->fmt == MQC_E2M1;
    if (nva == nullptr && !mxf4) {
        if ((st = check_workspace("conv2d_fwd", workspace, workspace_bytes,
                                  mqc_conv2d_fwd_workspace_bytes(c, xf, wf))) != MQC_OK)
            return st;
        uint8_t *wsp = static_cast<uint8_t *>(workspace);
        if ((st = gemm_operand(xq, xf, N, C, H, W, wsp, static_cast<cudaStream_t>(stream), ox)) != MQC_OK) return st;
        if ((st = gemm_operand(wq, wf, K, C, R, S, wsp, static_cast<cudaStream_t>(stream), ow)) != MQC_OK) return st;
    } else {
        // NVFP4: the packed codes themselves; a row of C padded to 32 codes is
        // round32(C) / 2 bytes, and the K-blocks below are 32 bytes (64 codes)
        ox.codes = static_cast<const uint8_t *>(xq);
        ow.codes = static_cast<const uint8_t *>(wq);
        ox.mma_fmt = ow.mma_fmt = MQC_E2M1;
        ox.inner = ow.inner = round_up(C, 32) / 2;
    }
    const int64_t Cp = ox.inner, Cpw = ow.inner;   // padded channel extents of X and W rows (bytes)
    // narrow channels (one 16-byte code row: C <= 16 of an 8-bit format) and
    // a batch of 16: a pixel's codes of the whole batch are one contiguous
    // 256-byte run, and an A box of 8 such runs is a whole tile (rows n
    // fastest), instead of 128 separate 16-byte rows
    const bool narrow = nva == nullptr && !mxf4 && Cp == 16 && Cpw == 16 && N == 16;
    GemmParams G;
    memset(&G, 0, sizeof G);
    G.CB = static_cast<int32_t>(nb32(Cp));
    G.wkb = largest_wkb(G.CB);
    G.k16 = narrow ? 1 : 0;
    if (narrow && qo == nullptr) {
        G.bn = 16;
        G.bq = 8;
        G.bp = 1;
    } else if (qo == nullptr) {
        choose_rows(Q, P, N, G.bq, G.bp, G.bn);
    } else {
        // quantized output: rows n fastest, bn = 16 (a batch of at most 16)
        // or 32, so that the rows of one pixel are lanes of one warp; the
        // pixels of a tile: the fewest computed rows, then the longest run
        // along q
        G.bn = N <= 16 ? 16 : 32;
        const int pix = 128 / G.bn;
        G.bq = pix;
        G.bp = 1;
        for (int bq = pix / 2; bq >= 1; bq /= 2) {
            const int bp = pix / bq;
            if (ceil_div(Q, bq) * bq * ceil_div(P, bp) * bp < ceil_div(Q, G.bq) * G.bq * ceil_div(P, G.bp) * G.bp) {
                G.bq = bq;
                G.bp = bp;
            }
        }
    }
    G.BN = choose_bn(K);
    G.nb_atoms = static_cast<int32_t>(ceil_div(G.BN, 128));
    G.Ne = N;
    G.TQ = static_cast<int32_t>(ceil_div(Q, G.bq));
    G.TP = static_cast<int32_t>(ceil_div(P, G.bp));
    G.TN = static_cast<int32_t>(ceil_div(N, G.bn));
    G.NT = static_cast<int32_t>(ceil_div(K, G.BN));
    G.Ncols = K;
    G.a_st_h = sh;
    G.a_st_w = sw;
    G.idesc = nva    ? make_idesc_nvf4(128, G.BN)
              : mxf4 ? make_idesc_mxf4(128, G.BN)
                     : make_idesc_mx(mma_fmt(ox.mma_fmt), mma_fmt(ow.mma_fmt), 128, G.BN);
    // A: one map per stride phase; dims (C, W', H', N) so that rows run along q
    bool phase_ok[16] = {};
    for (int attempt = (qo || narrow) ? 1 : 0; attempt < 2; ++attempt) {
        G.rows_nfirst = attempt;
        st = MQC_OK;
        for (int a = 0; a < sh && st == MQC_OK; ++a)
            for (int b = 0; b < sw && st == MQC_OK; ++b) {
                const int64_t Hh = ceil_div(H - a, sh), Ww = ceil_div(W - b, sw);
                phase_ok[a * sw + b] = Hh > 0 && Ww > 0;
                if (!phase_ok[a * sw + b]) continue;
                const uint8_t *base = ox.codes + (int64_t(a) * W + b) * N * Cp;
                if (narrow) {
                    // (n and c as one 256-byte dimension, W', H') of phase (a, b)
                    const uint64_t dims[3] = {uint64_t(N) * Cp, uint64_t(Ww), uint64_t(Hh)};
                    const uint64_t strd[2] = {uint64_t(sw) * N * Cp, uint64_t(sh) * W * N * Cp};
                    const uint32_t box[3] = {uint32_t(N * Cp), uint32_t(G.bq), uint32_t(G.bp)};
                    st = encode_codes_map(&G.amap[a * sw + b], base, 3, dims, strd, box, 0);
                } else if (!G.rows_nfirst) {
                    const uint64_t dims[4] = {uint64_t(Cp), uint64_t(Ww), uint64_t(Hh), uint64_t(N)};
                    const uint64_t strd[3] = {uint64_t(sw) * N * Cp, uint64_t(sh) * W * N * Cp, uint64_t(Cp)};
                    const uint32_t box[4] = {uint32_t(32 * G.wkb), uint32_t(G.bq), uint32_t(G.bp), uint32_t(G.bn)};
                    st = encode_codes_map(&G.amap[a * sw + b], base, 4, dims, strd, box, G.wkb);
                } else {
                    const uint64_t dims[4] = {uint64_t(Cp), uint64_t(N), uint64_t(Ww), uint64_t(Hh)};
                    const uint64_t strd[3] = {uint64_t(Cp), uint64_t(sw) * N * Cp, uint64_t(sh) * W * N * Cp};
                    const uint32_t box[4] = {uint32_t(32 * G.wkb), uint32_t(G.bn), uint32_t(G.bq), uint32_t(G.bp)};
                    st = encode_codes_map(&G.amap[a * sw + b], base, 4, dims, strd, box, G.wkb);
                }
            }
        if (st == MQC_OK) break;
    }
    if (st != MQC_OK) return st;
    {
        const uint64_t dims[3] = {uint64_t(Cpw), uint64_t(K), uint64_t(R) * S};
        const uint64_t strd[2] = {uint64_t(Cpw), uint64_t(K) * Cpw};
        const uint32_t box[3] = {uint32_t(narrow ? 16 : 32 * G.wkb), uint32_t(box_rows(K, G.BN)), 1u};
        if ((st = encode_codes_map(&G.bmap[0], ow.codes, 3, dims, strd, box, narrow ? 0 : G.wkb)) != MQC_OK)
            return st;
    }
    G.ntaps = 0;
    for (int r = 0; r < R; ++r)
        for (int s = 0; s < S; ++s) {
            int dh, ph, dw, pw;
            split_tap(r - c->pad_h, sh, dh, ph);
            split_tap(s - c->pad_w, sw, dw, pw);
            ConvTap &T = G.taps[G.ntaps++];
            T.btap = static_cast<int16_t>(r * S + s);
            T.sf_dh = static_cast<int16_t>(r - c->pad_h);
            T.sf_dw = static_cast<int16_t>(s - c->pad_w);
            if (phase_ok[ph * sw + pw]) {
                T.map = static_cast<int16_t>(ph * sw + pw);
                T.dh = static_cast<int16_t>(dh);
                T.dw = static_cast<int16_t>(dw);
            } else {           // a phase with no rows: read far outside (zeros)
                T.map = 0;
                T.dh = T.dw = -30000;
                T.sf_dh = T.sf_dw = -30000;
            }
        }
    G.nph = 1;
    G.ph_tap0[0] = 0;
    G.ph_tkb[0] = G.ntaps * G.CB;
    G.ph_Qe[0] = Q;
    G.ph_Pe[0] = P;
    G.ph_out_base[0] = 0;
    for (int i = 0; i < sh * sw; ++i)          // unused phases get a valid copy (never read)
        if (!phase_ok[i]) G.amap[i] = G.amap[0];
    G.n_amaps = sh * sw;
    G.n_bmaps = 1;
    const int rowb = narrow ? 16 : 32 * G.wkb;     // shared-memory bytes of a row of a box
    G.a_box_bytes = rowb * G.bq * G.bp * G.bn;
    G.b_box_bytes = rowb * box_rows(K, G.BN);
    G.a_slab = 128;
    G.b_slab = G.BN;
    const bool sqx = xf->block == MQC_BLOCK_SQ32, sqw = wf->block == MQC_BLOCK_SQ32;
    // square X blocks: the 16 rows of a pixel share its scale byte
    G.sf_pix = narrow && sqx ? 1 : 0;
    // the staged fp32 epilogue stores 16-byte runs of q: 16-byte aligned rows
    G.ep_stage = narrow && qo == nullptr && Q % 4 == 0 && (reinterpret_cast<uintptr_t>(y) & 15u) == 0 ? 1 : 0;
    G.sfa.base = xs;
    G.sfa.pix_pitch = (sqx ? nb32(N) : N) * nb32(Cp);
    G.sfa.row_shift = sqx ? 5 : 0;
    G.sfa.row_pitch = static_cast<int32_t>(nb32(Cp));
    G.sfa.kb_pitch = 1;
    G.sfa.rows = N;
    G.sfa.H = H;
    G.sfa.W = W;
    G.sfb.base = ws;
    G.sfb.tap_pitch = (sqw ? nb32(K) : K) * nb32(Cp);
    G.sfb.row_shift = sqw ? 5 : 0;
    G.sfb.row_pitch = static_cast<int32_t>(nb32(Cp));
    G.sfb.kb_pitch = 1;
    G.sfb.rows = K;
    G.sf_vec4 = G.CB % 4 == 0 && G.sfa.pix_pitch % 4 == 0 && G.sfa.row_pitch % 4 == 0 &&
                (reinterpret_cast<uintptr_t>(xs) & 3u) == 0;
    G.sfb_vec4 = G.CB % 4 == 0 && G.sfb.tap_pitch % 4 == 0 && G.sfb.row_pitch % 4 == 0 &&
                 (reinterpret_cast<uintptr_t>(ws) & 3u) == 0;
    if (nva != nullptr) {
        // E4M3 scales per 16 channels: A16 [pix][n][nb16], SQ16 [pix][n/16][nb16]
        // (W: [tap][k or k/16][nb16]); a 32-byte K-block has 4 of them
        const int64_t nb = round_up(C, 32) / 16;
        const bool sqx16 = nva->x_block == MQC_NV_SQ16, sqw16 = nva->w_block == MQC_NV_SQ16;
        G.sfa.pix_pitch = (sqx16 ? ceil_div(N, 16) : N) * nb;
        G.sfa.row_shift = sqx16 ? 4 : 0;
        G.sfa.row_pitch = static_cast<int32_t>(nb);
        G.sfa.kb_pitch = 1;
        G.sfa.nblk = static_cast<int32_t>(nb);
        G.sfb.tap_pitch = (sqw16 ? ceil_div(K, 16) : K) * nb;
        G.sfb.row_shift = sqw16 ? 4 : 0;
        G.sfb.row_pitch = static_cast<int32_t>(nb);
        G.sfb.kb_pitch = 1;
        G.sfb.nblk = static_cast<int32_t>(nb);
        // whole 4-byte atoms per load: every pitch and the block count
        // multiples of 4 (then no block is past the row), aligned bases
        G.sf_vec4 = nb % 4 == 0 && G.sfa.pix_pitch % 4 == 0 && G.sfb.tap_pitch % 4 == 0 &&
                    (reinterpret_cast<uintptr_t>(xs) & 3u) == 0 && (reinterpret_cast<uintptr_t>(ws) & 3u) == 0;
        G.sfb_vec4 = 0;
        G.nv_tx = nva->x_tscale;
        G.nv_tw = nva->w_tscale;
        G.pk = 2;
    } else if (mxf4) {
        // E8M0 scales per 32 channels (the MX layout above); a 32-byte K-block
        // (64 codes) has 2 of them
        const int64_t nb = round_up(C, 32) / 32;     // (Cp above counts bytes here)
        G.sfa.pix_pitch = (sqx ? nb32(N) : N) * nb;
        G.sfa.row_pitch = static_cast<int32_t>(nb);
        G.sfa.kb_pitch = 1;
        G.sfa.nblk = static_cast<int32_t>(nb);
        G.sfb.tap_pitch = (sqw ? nb32(K) : K) * nb;
        G.sfb.row_pitch = static_cast<int32_t>(nb);
        G.sfb.kb_pitch = 1;
        G.sfb.nblk = static_cast<int32_t>(nb);
        // two K-blocks (4 scale bytes) per aligned load: an even number of
        // K-blocks per tap, pitches and the block count multiples of 4
        G.sf_vec4 = G.CB % 2 == 0 && nb % 4 == 0 && G.sfa.pix_pitch % 4 == 0 && G.sfb.tap_pitch % 4 == 0 &&
                    (reinterpret_cast<uintptr_t>(xs) & 3u) == 0 && (reinterpret_cast<uintptr_t>(ws) & 3u) == 0;
        G.sfb_vec4 = 0;
        G.pk = 1;
    }
    G.out = y;
    G.os_q = 1;
    G.os_p = Q;
    G.os_n = int64_t(K) * P * Q;
    G.os_c = int64_t(P) * Q;
    if (qo != nullptr) {
        int64_t Kp, Np_ba, Kp_ab, Np;
        padded(qo->yf->fmt, MQC_ORDER_BA, K, N, Kp, Np_ba);
        padded(qo->yf->fmt, MQC_ORDER_AB, K, N, Kp_ab, Np);
        G.q_codes = static_cast<uint8_t *>(qo->yq);
        G.q_codes_alt = static_cast<uint8_t *>(qo->yq_alt);
        G.q_scales = qo->ys;
        G.q_y = qo->y;
        G.q_fmt = qo->yf->fmt;
        G.q_sq = qo->yf->block == MQC_BLOCK_SQ32 ? 1 : 0;
        G.q_act = qo->act;
        G.q_emax = emax_elem(qo->yf->fmt);
        G.q_Kp = static_cast<int32_t>(Kp);
        G.q_Np = static_cast<int32_t>(Np);
        G.q_nbA = static_cast<int32_t>(nb32(Kp));
        G.q_nbB = static_cast<int32_t>(nb32(N));
        G.q_lanes = G.bn;
        G.out = nullptr;
    }
    G.num_units = G.TQ * G.TP * G.TN * G.NT;
    return launch_gemm<kConv>(G, *dv, static_cast<cudaStream_t>(stream));
}

extern "C" {

// ------------------------------------------------------------------ input gradient
// Input gradient of a strided convolution as one sub-pixel GEMM (see
// subpixel.cuh): used when the stride phases number 2 to 4, tile the input
// exactly (H, W multiples of the stride) and C is a multiple of 16 (columns
// of one phase come in 16s).  Measured on the YOLOv8n layers (3x3, stride 2):
// one launch with 4 x C columns instead of phase launches with C columns.
struct SubpixPlan {
    bool on = false;
    SubpixGeom g{};
    size_t codes_bytes = 0, scale_bytes = 0;
};

static SubpixPlan subpix_plan(const mqc_conv *c, const mqc_mx *wf) {
    SubpixPlan sp;
    const int sh = c->stride_h, sw = c->stride_w;
    if (sh * sw < 2 || sh * sw > kMaxPhases || c->H % sh != 0 || c->W % sw != 0 || c->C % 16 != 0) return sp;
    int dh0 = 1 << 30, dh1 = -(1 << 30), dw0 = 1 << 30, dw1 = -(1 << 30);
    for (int a = 0; a < sh; ++a)
        for (int r = 0; r < c->R; ++r) {
            const int t = a + c->pad_h - r;
            if ((t % sh + sh) % sh != 0) continue;
            dh0 = std::min(dh0, t / sh);
            dh1 = std::max(dh1, t / sh);
        }
    for (int a = 0; a < sw; ++a)
        for (int s = 0; s < c->S; ++s) {
            const int t = a + c->pad_w - s;
            if ((t % sw + sw) % sw != 0) continue;
            dw0 = std::min(dw0, t / sw);
            dw1 = std::max(dw1, t / sw);
        }
    if (dh0 > dh1 || dw0 > dw1 || (dh1 - dh0 + 1) * (dw1 - dw0 + 1) > kMaxTaps) return sp;
    int64_t Ap, Bp;
    padded(wf->fmt, wf->order, c->C, c->K, Ap, Bp);
    const int64_t kpw = wf->order == MQC_ORDER_BA ? Ap : Bp;
    const bool sqw = wf->block == MQC_BLOCK_SQ32;
    SubpixGeom &g = sp.g;
    g.C = c->C;
    g.Cs = sh * sw * c->C;
    g.R = c->R;
    g.S = c->S;
    g.sh = sh;
    g.sw = sw;
    g.ph = c->pad_h;
    g.pw = c->pad_w;
    g.dh0 = dh0;
    g.dw0 = dw0;
    g.Rs = dh1 - dh0 + 1;
    g.Ss = dw1 - dw0 + 1;
    g.kpw = static_cast<int32_t>(kpw);
    g.nkb = static_cast<int32_t>(nb32(kpw));
    g.w_kb_pitch = static_cast<int32_t>(sqw ? nb32(c->C) : c->C);
    g.w_tap_pitch = nb32(kpw) * g.w_kb_pitch;
    g.w_row_shift = sqw ? 5 : 0;
    const int64_t ntap = int64_t(g.Rs) * g.Ss;
    sp.codes_bytes = static_cast<size_t>(round_up(ntap * g.Cs * kpw, 256));
    sp.scale_bytes = static_cast<size_t>(round_up(ntap * g.nkb * g.Cs, 256));
    sp.on = kpw % 16 == 0;
    return sp;
}

size_t mqc_conv2d_bwd_data_workspace_bytes(const mqc_conv *c, const mqc_mx *wf, const mqc_mx *gf) {
    if (!conv_ok(c) || !mx_ok(wf) || !mx_ok(gf)) return 0;
    const SubpixPlan sp = subpix_plan(c, wf);
    return widened_bytes(wf, c->K, c->C, c->R, c->S) + widened_bytes(gf, c->N, c->K, conv_P(c), conv_Q(c)) +
           (sp.on ? sp.codes_bytes + sp.scale_bytes : 0);
}

mqc_status mqc_conv2d_bwd_data(const void *wq, const uint8_t *ws, const mqc_mx *wf, const void *gq, const uint8_t *gs,
                               const mqc_mx *gf, const mqc_conv *c, float *gx, void *workspace, size_t workspace_bytes,
                               void *stream) {
    if (!conv_ok(c) || gx == nullptr) return fail(MQC_ERR_INVALID, "conv2d_bwd_data: bad conv descriptor or null output");
    mqc_status st = check_gemm_operand("W", wq, ws, wf, MQC_ORDER_AB, false);
    if (st != MQC_OK) return st;
    st = check_gemm_operand("G_Y", gq, gs, gf, MQC_ORDER_BA, true);
    if (st != MQC_OK) return st;
    if (c->R * c->S > kMaxTaps) return fail(MQC_ERR_UNSUPPORTED, "conv2d_bwd_data: at most %d kernel taps", kMaxTaps);
    DevInfo *dv;
    if ((st = dev_info(dv)) != MQC_OK) return st;
    const int N = c->N, C = c->C, H = c->H, W = c->W, K = c->K, R = c->R, S = c->S;
    const int sh = c->stride_h, sw = c->stride_w, P = conv_P(c), Q = conv_Q(c);
    if ((st = check_workspace("conv2d_bwd_data", workspace, workspace_bytes,
                              mqc_conv2d_bwd_data_workspace_bytes(c, wf, gf))) != MQC_OK)
        return st;
    uint8_t *wsp = static_cast<uint8_t *>(workspace);
    const SubpixPlan sp = subpix_plan(c, wf);
    // both operands OCP MXFP4 and the per-phase plan: the packed codes go to
    // the tensor core as they are (kind::mxf4), no widening
    const bool mxf4 = !sp.on && wf->fmt == MQC_E2M1 && gf->fmt == MQC_E2M1;
    GemmOperand ow, og;
    if (!mxf4) {
        if ((st = gemm_operand(wq, wf, K, C, R, S, wsp, static_cast<cudaStream_t>(stream), ow)) != MQC_OK) return st;
        if ((st = gemm_operand(gq, gf, N, K, P, Q, wsp, static_cast<cudaStream_t>(stream), og)) != MQC_OK) return st;
    } else {
        ow.codes = static_cast<const uint8_t *>(wq);
        og.codes = static_cast<const uint8_t *>(gq);
        ow.mma_fmt = og.mma_fmt = MQC_E2M1;
        ow.inner = og.inner = round_up(K, 32) / 2;     // bytes of a row of K codes padded to 32
    }
    const int64_t Kp = og.inner, Kpw = ow.inner;   // padded output-channel extents of G_Y and W rows
    const bool sqg = gf->block == MQC_BLOCK_SQ32, sqw = wf->block == MQC_BLOCK_SQ32;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    if (sp.on) {
        if (ow.inner != sp.g.kpw) return fail(MQC_ERR_UNSUPPORTED, "conv2d_bwd_data: weight row padding mismatch");
        uint8_t *scodes = wsp, *sscales = wsp + sp.codes_bytes;
        const SubpixGeom &g = sp.g;
        const int64_t work = (int64_t(g.Rs) * g.Ss * g.Cs * g.kpw) / 16 + int64_t(g.Rs) * g.Ss * g.nkb * g.Cs;
        const int blocks = static_cast<int>(std::min<int64_t>(ceil_div(work, 256), int64_t(dv->sms) * 4));
        subpix_weights_kernel<<<blocks, 256, 0, strm>>>(ow.codes, ws, scodes, sscales, g);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "subpix_weights_kernel launch");
        const int ntap = g.Rs * g.Ss, Cs = g.Cs, Qs = W / sw, Ps = H / sh;
        GemmParams G;
        memset(&G, 0, sizeof G);
        G.CB = static_cast<int32_t>(nb32(Kp));
        G.wkb = largest_wkb(G.CB);
        G.sub = 1;
        choose_rows(Qs, Ps, N, G.bq, G.bp, G.bn);
        G.BN = choose_bn(Cs);
        G.nb_atoms = static_cast<int32_t>(ceil_div(G.BN, 128));
        G.Ne = N;
        G.TQ = static_cast<int32_t>(ceil_div(Qs, G.bq));
        G.TP = static_cast<int32_t>(ceil_div(Ps, G.bp));
        G.TN = static_cast<int32_t>(ceil_div(N, G.bn));
        G.NT = static_cast<int32_t>(ceil_div(Cs, G.BN));
        G.Ncols = Cs;
        G.a_st_h = 1;
        G.a_st_w = 1;
        G.idesc = make_idesc_mx(mma_fmt(og.mma_fmt), mma_fmt(ow.mma_fmt), 128, G.BN);
        st = MQC_ERR_CUDA;
        for (int attempt = 0; attempt < 2 && st != MQC_OK; ++attempt) {
            G.rows_nfirst = attempt;
            if (!G.rows_nfirst) {
                const uint64_t dims[4] = {uint64_t(Kp), uint64_t(Q), uint64_t(P), uint64_t(N)};
                const uint64_t strd[3] = {uint64_t(N) * Kp, uint64_t(Q) * N * Kp, uint64_t(Kp)};
                const uint32_t box[4] = {uint32_t(32 * G.wkb), uint32_t(G.bq), uint32_t(G.bp), uint32_t(G.bn)};
                st = encode_codes_map(&G.amap[0], og.codes, 4, dims, strd, box, G.wkb);
            } else {
                const uint64_t dims[4] = {uint64_t(Kp), uint64_t(N), uint64_t(Q), uint64_t(P)};
                const uint64_t strd[3] = {uint64_t(Kp), uint64_t(N) * Kp, uint64_t(Q) * N * Kp};
                const uint32_t box[4] = {uint32_t(32 * G.wkb), uint32_t(G.bn), uint32_t(G.bq), uint32_t(G.bp)};
                st = encode_codes_map(&G.amap[0], og.codes, 4, dims, strd, box, G.wkb);
            }
        }
        if (st != MQC_OK) return st;
        {
            const uint64_t dims[3] = {uint64_t(Kpw), uint64_t(Cs), uint64_t(ntap)};
            const uint64_t strd[2] = {uint64_t(Kpw), uint64_t(Cs) * Kpw};
            const uint32_t box[3] = {uint32_t(32 * G.wkb), uint32_t(box_rows(Cs, G.BN)), 1u};
            if ((st = encode_codes_map(&G.bmap[0], scodes, 3, dims, strd, box, G.wkb)) != MQC_OK) return st;
        }
        G.ntaps = ntap;
        for (int t = 0; t < ntap; ++t) {
            ConvTap &T = G.taps[t];
            T.dh = T.sf_dh = static_cast<int16_t>(g.dh0 + t / g.Ss);
            T.dw = T.sf_dw = static_cast<int16_t>(g.dw0 + t % g.Ss);
            T.map = 0;
            T.aw = 0;
            T.btap = static_cast<int16_t>(t);
        }
        G.nph = 1;
        G.ph_tap0[0] = 0;
        G.ph_tkb[0] = ntap * G.CB;
        G.ph_Pe[0] = Ps;
        G.ph_Qe[0] = Qs;
        G.ph_out_base[0] = 0;
        G.n_amaps = 1;
        G.n_bmaps = 1;
        G.a_box_bytes = 32 * G.wkb * G.bq * G.bp * G.bn;
        G.b_box_bytes = 32 * G.wkb * box_rows(Cs, G.BN);
        G.a_slab = 128;
        G.b_slab = G.BN;
        G.sfa.base = gs;
        G.sfa.pix_pitch = (sqg ? nb32(N) : N) * nb32(Kp);
        G.sfa.row_shift = sqg ? 5 : 0;
        G.sfa.row_pitch = static_cast<int32_t>(nb32(Kp));
        G.sfa.kb_pitch = 1;
        G.sfa.rows = N;
        G.sfa.H = P;
        G.sfa.W = Q;
        G.sfb.base = sscales;
        G.sfb.tap_pitch = int64_t(g.nkb) * Cs;
        G.sfb.row_shift = 0;
        G.sfb.row_pitch = 1;
        G.sfb.kb_pitch = Cs;
        G.sfb.rows = Cs;
        G.sf_vec4 = G.CB % 4 == 0 && G.sfa.pix_pitch % 4 == 0 && G.sfa.row_pitch % 4 == 0 &&
                    (reinterpret_cast<uintptr_t>(gs) & 3u) == 0;
        G.sfb_vec4 = false;
        G.out = gx;
        G.os_q = sw;
        G.os_p = int64_t(sh) * W;
        G.os_n = int64_t(C) * H * W;
        G.os_c = int64_t(H) * W;
        // width phases stored in pairs when the column tiles hold whole pairs
        G.d2s = sw == 2 && G.BN % (2 * C) == 0 && (reinterpret_cast<uintptr_t>(gx) & 7u) == 0 ? 2 : 1;
        G.cpad = C;
        for (int a = 0; a < sh; ++a)
            for (int b = 0; b < sw; ++b) G.d2s_off[a * sw + b] = int64_t(a) * W + b;
        G.num_units = G.TQ * G.TP * G.TN * G.NT;
        return launch_gemm<kConv>(G, *dv, strm);
    }
    // output stride phases (ah, aw) with at least one row; the first one has
    // the largest extents and sets the tiling shared by a launch
    if (sh > 64 || sw > 64) return fail(MQC_ERR_UNSUPPORTED, "conv2d_bwd_data: stride above 64");
    // Output rows h = sh * p' + ah split into sh phases (their tap rows r
    // differ).  Along the width the sw phases share a tile: its rows
    // interleave them (sub = sw), so every output row is written whole.
    const int sub = sw;
    const int Qw = static_cast<int>(ceil_div(W, sw));     // q' extent (output column w = sw * q' + aw)
    const int Pe0 = static_cast<int>(ceil_div(H, sh));
    for (int first = 0; first < sh && first < H; first += kMaxPhases) {
        const int nph = std::min({kMaxPhases, sh - first, H - first});
        GemmParams G;
        memset(&G, 0, sizeof G);
        G.CB = static_cast<int32_t>(nb32(Kp));
        G.wkb = largest_wkb(G.CB);
        G.sub = sub;
        choose_rows(Qw, Pe0, N, G.bq, G.bp, G.bn, 128 / sub);
        G.BN = choose_bn(C);
        G.nb_atoms = static_cast<int32_t>(ceil_div(G.BN, 128));
        G.Ne = N;
        G.TQ = static_cast<int32_t>(ceil_div(Qw, G.bq));
        G.TP = static_cast<int32_t>(ceil_div(Pe0, G.bp));
        G.TN = static_cast<int32_t>(ceil_div(N, G.bn));
        G.NT = static_cast<int32_t>(ceil_div(C, G.BN));
        G.Ncols = C;
        G.a_st_h = 1;
        G.a_st_w = 1;
        G.idesc = make_idesc_mx(mma_fmt(og.mma_fmt), mma_fmt(ow.mma_fmt), 128, G.BN);
        st = MQC_ERR_CUDA;
        if (sub > 1) {
            // (C, slot, q, p, n): the slot dimension has extent 1 and a box of
            // sub, so a tap's box fills only the rows of its own slot
            G.rows_nfirst = 0;
            const uint64_t dims[5] = {uint64_t(Kp), 1u, uint64_t(Q), uint64_t(P), uint64_t(N)};
            const uint64_t strd[4] = {uint64_t(Kp), uint64_t(N) * Kp, uint64_t(Q) * N * Kp, uint64_t(Kp)};
            const uint32_t box[5] = {uint32_t(32 * G.wkb), uint32_t(sub), uint32_t(G.bq), uint32_t(G.bp),
                                     uint32_t(G.bn)};
            st = encode_codes_map(&G.amap[0], og.codes, 5, dims, strd, box, G.wkb);
        } else {
            for (int attempt = 0; attempt < 2 && st != MQC_OK; ++attempt) {
                G.rows_nfirst = attempt;
                if (!G.rows_nfirst) {
                    const uint64_t dims[4] = {uint64_t(Kp), uint64_t(Q), uint64_t(P), uint64_t(N)};
                    const uint64_t strd[3] = {uint64_t(N) * Kp, uint64_t(Q) * N * Kp, uint64_t(Kp)};
                    const uint32_t box[4] = {uint32_t(32 * G.wkb), uint32_t(G.bq), uint32_t(G.bp), uint32_t(G.bn)};
                    st = encode_codes_map(&G.amap[0], og.codes, 4, dims, strd, box, G.wkb);
                } else {
                    const uint64_t dims[4] = {uint64_t(Kp), uint64_t(N), uint64_t(Q), uint64_t(P)};
                    const uint64_t strd[3] = {uint64_t(Kp), uint64_t(N) * Kp, uint64_t(Q) * N * Kp};
                    const uint32_t box[4] = {uint32_t(32 * G.wkb), uint32_t(G.bn), uint32_t(G.bq), uint32_t(G.bp)};
                    st = encode_codes_map(&G.amap[0], og.codes, 4, dims, strd, box, G.wkb);
                }
            }
        }
        if (st != MQC_OK) return st;
        {
            const uint64_t dims[3] = {uint64_t(Kpw), uint64_t(C), uint64_t(R) * S};
            const uint64_t strd[2] = {uint64_t(Kpw), uint64_t(C) * Kpw};
            const uint32_t box[3] = {uint32_t(32 * G.wkb), uint32_t(box_rows(C, G.BN)), 1u};
            if ((st = encode_codes_map(&G.bmap[0], ow.codes, 3, dims, strd, box, G.wkb)) != MQC_OK) return st;
        }
        // taps of phase ah: kernel rows r with (ah + pad - r) divisible by sh,
        // every kernel column s; tap (r, s) feeds slot aw = (s - pad) mod sw
        G.ntaps = 0;
        G.nph = nph;
        for (int k = 0; k < nph; ++k) {
            const int ah = first + k;
            G.ph_tap0[k] = G.ntaps;
            for (int r = 0; r < R; ++r) {
                if (((ah + c->pad_h - r) % sh + sh) % sh != 0) continue;
                const int dr = (ah + c->pad_h - r) / sh;
                for (int s = 0; s < S; ++s) {
                    const int aw = ((s - c->pad_w) % sw + sw) % sw;
                    const int ds = (aw + c->pad_w - s) / sw;
                    ConvTap &T = G.taps[G.ntaps++];
                    T.dh = T.sf_dh = static_cast<int16_t>(dr);
                    T.dw = T.sf_dw = static_cast<int16_t>(ds);
                    T.map = 0;
                    T.aw = static_cast<int16_t>(aw);
                    T.btap = static_cast<int16_t>(r * S + s);
                }
            }
            G.ph_tkb[k] = (G.ntaps - G.ph_tap0[k]) * G.CB;
            G.ph_Pe[k] = static_cast<int32_t>(ceil_div(H - ah, sh));
            G.ph_Qe[k] = W;                      // limit of the output column sw * q' + aw
            G.ph_out_base[k] = int64_t(ah) * W;
        }
        G.n_amaps = 1;
        G.n_bmaps = 1;
        G.a_box_bytes = 32 * G.wkb * sub * G.bq * G.bp * G.bn;
        G.b_box_bytes = 32 * G.wkb * box_rows(C, G.BN);
        G.a_slab = 128;
        G.b_slab = G.BN;
        G.sfa.base = gs;
        G.sfa.pix_pitch = (sqg ? nb32(N) : N) * nb32(Kp);
        G.sfa.row_shift = sqg ? 5 : 0;
        G.sfa.row_pitch = static_cast<int32_t>(nb32(Kp));
        G.sfa.kb_pitch = 1;
        G.sfa.rows = N;
        G.sfa.H = P;
        G.sfa.W = Q;
        G.sfb.base = ws;
        G.sfb.tap_pitch = nb32(Kp) * (sqw ? nb32(C) : C);
        G.sfb.row_shift = sqw ? 5 : 0;
        G.sfb.row_pitch = 1;
        G.sfb.kb_pitch = static_cast<int32_t>(sqw ? nb32(C) : C);
        G.sfb.rows = C;
        G.sf_vec4 = G.CB % 4 == 0 && G.sfa.pix_pitch % 4 == 0 && G.sfa.row_pitch % 4 == 0 &&
                    (reinterpret_cast<uintptr_t>(gs) & 3u) == 0;
        G.sfb_vec4 = false;   // the weights' scales run along K with a stride of C per block
        if (mxf4) {
            // scales per 32 output channels: G_Y [pix][n or n/32][nbK] (blocks
            // adjacent), W [tap][nbK][C or C/32] (blocks C or C/32 apart)
            const int64_t nbK = round_up(K, 32) / 32;
            G.idesc = make_idesc_mxf4(128, G.BN);
            G.sfa.pix_pitch = (sqg ? nb32(N) : N) * nbK;
            G.sfa.row_pitch = static_cast<int32_t>(nbK);
            G.sfa.kb_pitch = 1;
            G.sfa.nblk = static_cast<int32_t>(nbK);
            G.sfb.tap_pitch = nbK * (sqw ? nb32(C) : C);
            G.sfb.kb_pitch = static_cast<int32_t>(sqw ? nb32(C) : C);
            G.sfb.nblk = static_cast<int32_t>(nbK);
            // aligned 4-byte loads of the A scales (two K-blocks) when every
            // tap has an even number of K-blocks and the pitches allow
            G.sf_vec4 = G.CB % 2 == 0 && nbK % 4 == 0 && G.sfa.pix_pitch % 4 == 0 &&
                        (reinterpret_cast<uintptr_t>(gs) & 3u) == 0;
            G.pk = 1;
        }
        G.out = gx;
        G.os_q = 1;
        G.os_p = int64_t(sh) * W;
        G.os_n = int64_t(C) * H * W;
        G.os_c = int64_t(H) * W;
        G.num_units = G.TQ * G.TP * G.TN * G.nph * G.NT;
        if ((st = launch_gemm<kConv>(G, *dv, strm)) != MQC_OK) return st;
    }
    return MQC_OK;
}

// ------------------------------------------------------------------ weight gradient
// Weight-gradient tiling.  With at most 128 input channels the kernel taps
// join the GEMM columns: a unit covers ntg taps x cpad channel rows (cpad =
// C rounded up to 8, at most 256 columns), so one MMA per K-block serves all
// of them instead of one narrow MMA per tap.
struct WgradPlan {
    int BN, splits, ntg, ngroups, cpad;
    bool wbox;      // tap groups of whole kernel rows, loaded as window boxes
    int64_t kiters;
};

static WgradPlan wgrad_plan(const mqc_conv *c, const DevInfo &d) {
    WgradPlan w{};
    const int P = conv_P(c), Q = conv_Q(c);
    const int64_t Np = round_up(c->N, 16);
    const int64_t NB = nb32(Np);
    const int wkb = largest_wkb(NB);
    const int bqk = 4 / wkb;
    const int ntaps = c->R * c->S;
    w.kiters = int64_t(P) * ceil_div(Q, bqk) * (NB / wkb);
    w.cpad = static_cast<int>(round_up(c->C, 8));
    const int most = std::max(1, 256 / w.cpad);   // taps whose columns fit 256
    if (ntaps > 1 && c->C <= 128 && most >= c->S) {
        // groups of kr whole kernel rows: one TMA box per pixel brings every
        // (tap, channel) row of the group (the taps of a kernel row are
        // neighbouring pixels of X, whatever the stride).  kr: the fewest GEMM
        // columns over all groups (a partial last group still computes whole
        // rows), then the fewest groups.  Measured on the YOLOv8n layers:
        // C = 16 one group of 3 rows, C = 32 three groups of one row.
        int kr = 1;
        for (int k = 1; k <= std::min(c->R, most / c->S); ++k)
            if (ceil_div(c->R, k) * round_up(c->S * k * w.cpad, 16) <=
                ceil_div(c->R, kr) * round_up(c->S * kr * w.cpad, 16))
                kr = k;
        w.ngroups = static_cast<int>(ceil_div(c->R, kr));
        w.ntg = c->S * kr;
        w.wbox = true;
        w.BN = static_cast<int>(round_up(w.ntg * w.cpad, 16));
    } else if (ntaps > 1 && c->C <= 128) {
        w.ngroups = static_cast<int>(ceil_div(ntaps, most));
        w.ntg = static_cast<int>(ceil_div(ntaps, w.ngroups));
        w.BN = static_cast<int>(round_up(w.ntg * w.cpad, 16));
    } else {
        w.ntg = 1;
        w.ngroups = ntaps;
        w.BN = choose_bn(c->C);
    }
    const int64_t base = ceil_div(c->K, 128) * ceil_div(c->C, w.ntg > 1 ? c->C : w.BN) * int64_t(w.ngroups);
    int64_t sp = base >= d.sms ? 1 : d.sms / base;
    sp = std::min<int64_t>(sp, std::max<int64_t>(1, w.kiters / 8));
    w.splits = static_cast<int>(std::max<int64_t>(1, sp));
    return w;
}

// Split-K partial sums (when the reduction is split) at the start of the
// workspace, then the widened copies of E2M1 operands.
static size_t wgrad_partial_bytes(const mqc_conv *c, const WgradPlan &w) {
    if (w.splits <= 1) return 0;
    return static_cast<size_t>(round_up(int64_t(w.splits) * c->K * c->C * c->R * c->S * int64_t(sizeof(float)), 256));
}

size_t mqc_conv2d_bwd_weight_workspace_bytes(const mqc_conv *c, const mqc_mx *gf, const mqc_mx *xf) {
    if (!conv_ok(c) || !mx_ok(gf) || !mx_ok(xf)) return 0;
    DevInfo *dv;
    if (dev_info(dv) != MQC_OK) return 0;
    const WgradPlan w = wgrad_plan(c, *dv);
    return wgrad_partial_bytes(c, w) + widened_bytes(gf, c->N, c->K, conv_P(c), conv_Q(c)) +
           widened_bytes(xf, c->N, c->C, c->H, c->W);
}

mqc_status mqc_conv2d_bwd_weight(const void *gq, const uint8_t *gs, const mqc_mx *gf, const void *xq,
                                 const uint8_t *xs, const mqc_mx *xf, const mqc_conv *c, float *gw, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    if (!conv_ok(c) || gw == nullptr) return fail(MQC_ERR_INVALID, "conv2d_bwd_weight: bad conv descriptor or null output");
    mqc_status st = check_gemm_operand("G_Y", gq, gs, gf, MQC_ORDER_AB, false);
    if (st != MQC_OK) return st;
    st = check_gemm_operand("X", xq, xs, xf, MQC_ORDER_AB, false);
    if (st != MQC_OK) return st;
    if (c->R * c->S > kMaxTaps) return fail(MQC_ERR_UNSUPPORTED, "conv2d_bwd_weight: at most %d kernel taps", kMaxTaps);
    // one activation tensor map per stride phase, four at most
    if (c->stride_h * c->stride_w > 4) return fail(MQC_ERR_UNSUPPORTED, "conv2d_bwd_weight: stride product above 4");
    DevInfo *dv;
    if ((st = dev_info(dv)) != MQC_OK) return st;
    const int N = c->N, C = c->C, H = c->H, W = c->W, K = c->K, R = c->R, S = c->S;
    const int sh = c->stride_h, sw = c->stride_w, P = conv_P(c), Q = conv_Q(c);
    GemmParams G;
    memset(&G, 0, sizeof G);
    const WgradPlan plan = wgrad_plan(c, *dv);
    const int64_t kiters = plan.kiters;
    G.BN = plan.BN;
    G.splits = plan.splits;
    G.ntg = plan.ntg;
    G.ngroups = plan.ngroups;
    G.cpad = plan.cpad;
    if ((st = check_workspace("conv2d_bwd_weight", workspace, workspace_bytes,
                              mqc_conv2d_bwd_weight_workspace_bytes(c, gf, xf))) != MQC_OK)
        return st;
    uint8_t *wsp = static_cast<uint8_t *>(workspace) + wgrad_partial_bytes(c, plan);
    GemmOperand og, ox;
    if ((st = gemm_operand(gq, gf, N, K, P, Q, wsp, static_cast<cudaStream_t>(stream), og)) != MQC_OK) return st;
    if ((st = gemm_operand(xq, xf, N, C, H, W, wsp, static_cast<cudaStream_t>(stream), ox)) != MQC_OK) return st;
    const int64_t Np = og.inner, Npx = ox.inner;   // padded batch extents of G_Y and X rows
    const int64_t NB = nb32(Np);
    G.wkb = largest_wkb(NB);
    G.bqk = 4 / G.wkb;
    G.NC = static_cast<int32_t>(NB / G.wkb);
    G.QG = static_cast<int32_t>(ceil_div(Q, G.bqk));
    G.kiters_total = static_cast<int32_t>(kiters);
    G.P = P;
    G.Q = Q;
    G.nb_atoms = static_cast<int32_t>(ceil_div(G.BN, 128));
    G.MT = static_cast<int32_t>(ceil_div(K, 128));
    G.NT = G.ntg > 1 ? 1 : static_cast<int32_t>(ceil_div(C, G.BN));
    G.Mrows = K;
    G.Ncols = C;
    G.x_st_h = sh;
    G.x_st_w = sw;
    G.idesc = make_idesc_mx(mma_fmt(og.mma_fmt), mma_fmt(ox.mma_fmt), 128, G.BN);
    // batch of at most 16 (rows of 16 codes) and channel counts in 16s: the
    // maps take 16 rows of 16 bytes as one 256-byte row, unswizzled
    G.k16 = Np == 16 && Npx == 16 && K % 16 == 0 && C % 16 == 0 && G.wkb == 1;
    const int rb = G.k16 ? 16 : 32 * G.wkb;   // bytes of one operand row of a box
    if (G.k16) {
        const uint64_t dims[4] = {256, uint64_t(K / 16), uint64_t(Q), uint64_t(P)};
        const uint64_t strd[3] = {256, uint64_t(K) * 16, uint64_t(Q) * K * 16};
        const uint32_t box[4] = {256, uint32_t(box_rows(K, 128) / 16), uint32_t(G.bqk), 1u};
        if ((st = encode_codes_map(&G.amap[0], og.codes, 4, dims, strd, box, 0)) != MQC_OK) return st;
    } else {
        const uint64_t dims[4] = {uint64_t(Np), uint64_t(K), uint64_t(Q), uint64_t(P)};
        const uint64_t strd[3] = {uint64_t(Np), uint64_t(K) * Np, uint64_t(Q) * K * Np};
        const uint32_t box[4] = {uint32_t(32 * G.wkb), uint32_t(box_rows(K, 128)), uint32_t(G.bqk), 1u};
        if ((st = encode_codes_map(&G.amap[0], og.codes, 4, dims, strd, box, G.wkb)) != MQC_OK) return st;
    }
    G.wbox = plan.wbox;
    G.wb_S = S;
    G.wb_ph = c->pad_h;
    G.wb_pw = c->pad_w;
    bool phase_ok[16] = {};
    for (int a = 0; a < sh; ++a)
        for (int b = 0; b < sw; ++b) {
            const int64_t Hh = ceil_div(H - a, sh), Ww = ceil_div(W - b, sw);
            phase_ok[a * sw + b] = Hh > 0 && Ww > 0;
            if (!phase_ok[a * sw + b]) continue;
            const uint8_t *base = ox.codes + (int64_t(a) * W + b) * C * Npx;
            const int rows = G.ntg > 1 ? G.cpad : box_rows(C, G.BN);
            // one tap: a box over the kit's bqk pixels; tap groups: one pixel
            // of one tap per box (cpad rows), placed at that tap's rows
            const uint32_t box[4] = {uint32_t(G.k16 ? 256 : 32 * G.wkb), uint32_t(G.k16 ? rows / 16 : rows),
                                     uint32_t(G.ntg > 1 ? 1 : G.bqk), 1u};
            if (G.k16) {
                const uint64_t dims[4] = {256, uint64_t(C / 16), uint64_t(Ww), uint64_t(Hh)};
                const uint64_t strd[3] = {256, uint64_t(sw) * C * 16, uint64_t(sh) * W * C * 16};
                if ((st = encode_codes_map(&G.bmap[a * sw + b], base, 4, dims, strd, box, 0)) != MQC_OK) return st;
            } else {
                const uint64_t dims[4] = {uint64_t(Npx), uint64_t(C), uint64_t(Ww), uint64_t(Hh)};
                const uint64_t strd[3] = {uint64_t(Npx), uint64_t(sw) * C * Npx, uint64_t(sh) * W * C * Npx};
                if ((st = encode_codes_map(&G.bmap[a * sw + b], base, 4, dims, strd, box, G.wkb)) != MQC_OK)
                    return st;
            }
        }
    G.ntaps = 0;
    for (int r = 0; r < R; ++r)
        for (int s = 0; s < S; ++s) {
            int dh, ph, dw, pw;
            split_tap(r - c->pad_h, sh, dh, ph);
            split_tap(s - c->pad_w, sw, dw, pw);
            ConvTap &T = G.taps[G.ntaps++];
            T.btap = static_cast<int16_t>(r * S + s);
            T.sf_dh = static_cast<int16_t>(r - c->pad_h);
            T.sf_dw = static_cast<int16_t>(s - c->pad_w);
            if (phase_ok[ph * sw + pw]) {
                T.map = static_cast<int16_t>(ph * sw + pw);
                T.dh = static_cast<int16_t>(dh);
                T.dw = static_cast<int16_t>(dw);
            } else {
                T.map = 0;
                for (int i = 0; i < sh * sw; ++i)
                    if (phase_ok[i]) { T.map = static_cast<int16_t>(i); break; }
                T.dh = T.dw = -30000;
                T.sf_dh = T.sf_dw = -30000;
            }
        }
    for (int i = 0; i < sh * sw; ++i)
        if (!phase_ok[i])
            for (int j = 0; j < sh * sw; ++j)
                if (phase_ok[j]) { G.bmap[i] = G.bmap[j]; break; }
    G.n_amaps = 1;
    G.n_bmaps = sh * sw;
    if (G.wbox) {
        // (batch, C, W, H) of the whole X; a box of cpad channels x S x kr pixels
        const uint64_t dims[4] = {G.k16 ? 256 : uint64_t(Npx), uint64_t(G.k16 ? C / 16 : C), uint64_t(W), uint64_t(H)};
        const uint64_t strd[3] = {G.k16 ? 256 : uint64_t(Npx), uint64_t(C) * Npx, uint64_t(W) * C * Npx};
        const uint32_t box[4] = {uint32_t(G.k16 ? 256 : 32 * G.wkb), uint32_t(G.k16 ? G.cpad / 16 : G.cpad),
                                 uint32_t(S), uint32_t(G.ntg / S)};
        if ((st = encode_codes_map(&G.bmap[0], ox.codes, 4, dims, strd, box, G.k16 ? 0 : G.wkb)) != MQC_OK)
            return st;
        G.n_bmaps = 1;
    }
    G.a_slab = box_rows(K, 128);
    G.b_slab = G.ntg > 1 ? G.BN : box_rows(C, G.BN);
    G.a_box_bytes = rb * G.a_slab * G.bqk;
    G.b_box_bytes = G.wbox ? rb * G.cpad * G.ntg : (G.ntg > 1 ? rb * G.cpad : rb * G.b_slab * G.bqk);
    const bool sqg = gf->block == MQC_BLOCK_SQ32, sqx = xf->block == MQC_BLOCK_SQ32;
    G.sfa.base = gs;
    G.sfa.pix_pitch = nb32(Np) * (sqg ? nb32(K) : K);
    G.sfa.kb_pitch = static_cast<int32_t>(sqg ? nb32(K) : K);
    G.sfa.row_shift = sqg ? 5 : 0;
    G.sfa.row_pitch = 1;
    G.sfa.rows = K;
    G.sfa.H = P;
    G.sfa.W = Q;
    G.sfb.base = xs;
    G.sfb.pix_pitch = nb32(Np) * (sqx ? nb32(C) : C);
    G.sfb.kb_pitch = static_cast<int32_t>(sqx ? nb32(C) : C);
    G.sfb.row_shift = sqx ? 5 : 0;
    G.sfb.row_pitch = 1;
    G.sfb.rows = C;
    G.sfb.H = H;
    G.sfb.W = W;
    // square blocks on both sides and every 16-column group of an atom inside
    // one tap: one scale per 16-row group (columns start at multiples of 16)
    G.sq_gather = sqg && sqx && (G.ntg == 1 || G.cpad % 16 == 0);
    G.sq16 = G.ntg > 1 ? G.cpad % 32 != 0 : G.BN % 32 != 0 && G.NT > 1;
    G.out = G.splits > 1 ? static_cast<float *>(workspace) : gw;
    G.out_base = 0;
    G.os_m = int64_t(C) * R * S;
    G.os_c = int64_t(R) * S;
    G.split_pitch = int64_t(K) * C * R * S;
    G.num_units = G.MT * G.NT * G.ngroups * G.splits;
    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    if ((st = launch_gemm<kWgrad>(G, *dv, strm)) != MQC_OK) return st;
    if (G.splits > 1) {
        const int64_t n = int64_t(K) * C * R * S;
        const int blocks = static_cast<int>(std::min<int64_t>(ceil_div(n, 128), int64_t(dv->sms) * 16));
        splitk_reduce_kernel<<<blocks, 128, 0, strm>>>(static_cast<const float *>(workspace), gw, n, G.splits);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "splitk_reduce_kernel launch");
    }
    return MQC_OK;
}

// ------------------------------------------------------------------ weight gradient, no allocation
// Split-K scratch owned by the library: one copy per device, alive until the
// process exits.  Host code must not use the symbol itself as a device
// address; it looks the address up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MQC_NOALLOC_SCRATCH_BYTES];

static std::mutex g_noalloc_mu;
static void *g_noalloc_ptr[64];

mqc_status mqc_conv2d_bwd_weight_noalloc(const void *gq, const uint8_t *gs, const mqc_mx *gf, const void *xq,
                                         const uint8_t *xs, const mqc_mx *xf, const mqc_conv *c, float *gw,
                                         void *stream) {
    if (!conv_ok(c) || gw == nullptr)
        return fail(MQC_ERR_INVALID, "conv2d_bwd_weight_noalloc: bad conv descriptor or null output");
    mqc_status st = check_gemm_operand("G_Y", gq, gs, gf, MQC_ORDER_AB, false);
    if (st != MQC_OK) return st;
    st = check_gemm_operand("X", xq, xs, xf, MQC_ORDER_AB, false);
    if (st != MQC_OK) return st;
    const size_t need = mqc_conv2d_bwd_weight_workspace_bytes(c, gf, xf);
    if (need > MQC_NOALLOC_SCRATCH_BYTES)
        return fail(MQC_ERR_WORKSPACE,
                    "conv2d_bwd_weight_noalloc: needs %zu bytes of split-K scratch, above the %u-byte static "
                    "maximum; use mqc_conv2d_bwd_weight with a workspace",
                    need, MQC_NOALLOC_SCRATCH_BYTES);
    void *scratch = nullptr;
    if (need > 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
        if (dev < 0 || dev >= 64) return fail(MQC_ERR_CUDA, "device ordinal %d out of range", dev);
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        if (g_noalloc_ptr[dev] == nullptr) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(split-K scratch)");
            g_noalloc_ptr[dev] = p;
        }
        scratch = g_noalloc_ptr[dev];
    }
    return mqc_conv2d_bwd_weight(gq, gs, gf, xq, xs, xf, c, gw, scratch, scratch ? MQC_NOALLOC_SCRATCH_BYTES : 0,
                                 stream);
}

// ------------------------------------------------------------------ status
mqc_status mqc_get_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, g_mqc_device_error, sizeof v);
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    if (v != 0) {
        e = cudaMemcpyToSymbol(g_mqc_device_error, &zero, sizeof zero);
        if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
        return fail(MQC_ERR_DEVICE_TIMEOUT, "a kernel-side wait ran out of time (device error %d)", v);
    }
    return MQC_OK;
}

mqc_status mqc_debug_expire_wait(int64_t limit_ns, void *stream) {
    if (limit_ns < 1000 || limit_ns > 10000000000ll) return fail(MQC_ERR_INVALID, "limit_ns out of range");
    DevInfo *dv;
    mqc_status st = dev_info(dv);
    if (st != MQC_OK) return st;
    expire_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_ns));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "expire_wait_kernel launch");
    return MQC_OK;
}

}  // extern "C"
