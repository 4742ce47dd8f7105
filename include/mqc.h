/*
 * mqc.h -- C ABI of libmqc, a B200 (sm_100a) implementation of the MicroQonv
 * hot path ("MicroQonv: Reshaping Convolution Tensors for Efficient
 * Microscaling in Training and Inference", arXiv:2609.28358):
 *
 *   1. single-pass OCP-MX quantization of the convolution tensors X, W and
 *      G_Y into the channel-batch-first layout        -> mqc_quantize_mx
 *   2. channel-batch-first im2col on quantized codes  -> mqc_im2col_cbf
 *      (explicit form; the GEMMs below fold it into their shared-memory
 *      staging and never write the expansion)
 *   3. block-scaled tensor-core GEMMs of the convolution forward pass, the
 *      input gradient and the weight gradient         -> mqc_conv2d_fwd,
 *                                                        mqc_conv2d_bwd_data,
 *                                                        mqc_conv2d_bwd_weight
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Memory: every tensor pointer is a DEVICE pointer owned by the caller.
 *   The library never allocates, frees or retains device memory.  Buffers must
 *   be 16-byte aligned (else MQC_ERR_ALIGNMENT).  Sizes of quantized buffers
 *   come from mqc_codes_bytes / mqc_scales_bytes.
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *   default stream).  Every call only enqueues work on that stream and returns;
 *   results are ready when the stream is synchronized.
 * - Errors: arguments are validated on the host before anything is launched;
 *   a failed check returns a negative mqc_status and launches nothing.
 *   mqc_last_error_message() gives a one-line reason for the calling thread's
 *   last failure.  Kernel-side waits are bounded in time: a wait that runs out
 *   records MQC_ERR_DEVICE_TIMEOUT in a device flag that
 *   mqc_get_device_status() reads and clears.
 * - Shapes follow the paper's section II-A (PyTorch conventions):
 *   X [N][C][H][W], W [K][C][R][S], Y and G_Y [N][K][P][Q], with
 *   P = (H + 2*pad_h - R)/stride_h + 1 and Q likewise; convolution is
 *   cross-correlation with zero padding (Eq. 1-3).
 */
#ifndef MQC_H
#define MQC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MQC_API __attribute__((visibility("default")))
#else
#define MQC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MQC_OK = 0,
    MQC_ERR_INVALID = -1,        /* bad argument (null pointer, bad shape, bad enum) */
    MQC_ERR_UNSUPPORTED = -2,    /* valid request this build does not implement */
    MQC_ERR_CUDA = -3,           /* a CUDA runtime or driver call failed */
    MQC_ERR_DEVICE_TIMEOUT = -4, /* a bounded kernel-side wait ran out */
    MQC_ERR_ALIGNMENT = -5,      /* a pointer is not 16-byte aligned */
    MQC_ERR_WORKSPACE = -6       /* workspace missing or too small */
} mqc_status;

/* MX element formats (OCP MX v1.0): FP8 E4M3 (max 448), FP8 E5M2 (max 57344),
 * FP4 E2M1 (max 6).  Paper, section III-A (text of Eq. 4) names 448 and 6. */
typedef enum { MQC_E4M3 = 0, MQC_E5M2 = 1, MQC_E2M1 = 2 } mqc_fmt;

/* Quantization direction (paper, section IV-B).  Every tensor has an A-axis
 * and a B-axis, the reduction axes of the two GEMMs it takes part in:
 *     tensor   A-axis (d1)      B-axis (d0)
 *     X        C (forward)      N (weight gradient)
 *     W        C (forward)      K (input gradient)
 *     G_Y      K (input grad.)  N (weight gradient)
 * A32: 32 consecutive elements along A share one E8M0 scale; B32: along B;
 * SQ32: a 32x32 square over (B, A) shares one scale, so every 32-line in
 * either direction is a valid OCP block and the tensor is quantized once for
 * both of its GEMMs (the paper's square blocks at OCP's 32 granularity). */
typedef enum { MQC_BLOCK_A32 = 0, MQC_BLOCK_B32 = 1, MQC_BLOCK_SQ32 = 2 } mqc_block;

/* Code order inside one spatial position of the channel-batch-first layout
 * (paper, section IV-A, Fig. 3: each (h, w) holds a contiguous B x A block):
 * BA = A-axis innermost, AB = B-axis innermost. */
typedef enum { MQC_ORDER_BA = 0, MQC_ORDER_AB = 1 } mqc_order;

/* Which conv tensor a size query refers to. */
typedef enum { MQC_ROLE_X = 0, MQC_ROLE_W = 1, MQC_ROLE_G = 2 } mqc_role;

/* A 4-D fp32 source [d0][d1][d2][d3] with element strides (NCHW-like):
 * d0 = B-axis, d1 = A-axis, (d2, d3) = spatial. */
typedef struct { int32_t d0, d1, d2, d3; int64_t s0, s1, s2, s3; } mqc_t4;

typedef struct { int32_t fmt, block, order; } mqc_mx;

typedef struct {
    int32_t N, C, H, W;          /* input feature map X [N][C][H][W] */
    int32_t K, R, S;             /* weights W [K][C][R][S] */
    int32_t stride_h, stride_w, pad_h, pad_w;
} mqc_conv;

/* Quantized layout.  For a tensor with extents (d0=B, d1=A, d2, d3):
 *   order BA: codes[((h*d3 + w)*Bp + b)*Ap + a]      (Ap = A rounded up to a
 *             16-byte row: 16 FP8 codes or 32 FP4 codes; Bp = B)
 *   order AB: codes[((h*d3 + w)*Ap + a)*Bp + b]      (Bp rounded, Ap = A)
 * FP4 codes are packed two per byte, even element in the low nibble.  Padding
 * codes are +0.  One E8M0 scale byte per block, nb(x) = ceil(x/32):
 *   A32 : scales[(pix*Bp + b)*nb(Ap) + a/32]
 *   B32 : scales[(pix*nb(Bp) + b/32)*Ap + a]
 *   SQ32: scales[(pix*nb(Bp) + b/32)*nb(Ap) + a/32]      pix = h*d3 + w
 * Blocks that run past an axis end are short (they hold only real elements).
 * Returns -1 for invalid arguments. */
MQC_API int64_t mqc_codes_bytes(const mqc_mx *mx, int32_t d0, int32_t d1, int32_t d2, int32_t d3);
MQC_API int64_t mqc_scales_bytes(const mqc_mx *mx, int32_t d0, int32_t d1, int32_t d2, int32_t d3);

/* Extents (d0, d1, d2, d3) of X, W or G_Y for a convolution. */
MQC_API mqc_status mqc_tensor_dims(mqc_role role, const mqc_conv *conv, int32_t dims[4]);

/* MX quantization, one pass (paper, section III-A with the OCP MX shared
 * scale; directions of section IV-B; layout of section IV-A).
 *   src     fp32 device tensor described by `src_desc` (any element strides).
 *   mx      format, block mode and code order of `codes`.
 *   codes   device buffer of mqc_codes_bytes(mx, dims) bytes.
 *   scales  device buffer of mqc_scales_bytes(mx, dims) bytes.
 *   codes_alt  optional (may be NULL): a second copy of the SAME codes in the
 *           other order (AB if mx->order is BA and vice versa), written from
 *           the same read of `src`; its size is mqc_codes_bytes with the
 *           other order.  The scales are shared by both copies.
 * Per block: amax -> E8M0 scale 2^e with e = floor(log2 amax) - emax_elem
 * (clamped to [-127,127]; amax 0 -> 0x00; non-finite -> 0xFF), each element
 * x*2^-e rounded to nearest even with saturation to the largest finite code.
 * Errors: MQC_ERR_INVALID (bad extents/enums/null), MQC_ERR_ALIGNMENT. */
MQC_API mqc_status mqc_quantize_mx(const float *src, const mqc_t4 *src_desc, const mqc_mx *mx,
                           void *codes, uint8_t *scales, void *codes_alt, void *stream);

/* Several tensors quantized in ONE kernel launch, e.g. the weights of every
 * layer right after a weight update (the paper quantizes the weights once
 * per update, section V).  Element i of each array describes one tensor
 * exactly as the arguments of mqc_quantize_mx do; all tensors share the
 * format, block mode and code order in `mx`; codes_alt is NULL or an array
 * whose every entry is a buffer (a second code order for all tensors).
 * The results are those of count separate mqc_quantize_mx calls.
 *   count   1 .. 16.
 * Errors: as mqc_quantize_mx, for the first tensor that fails its checks. */
MQC_API mqc_status mqc_quantize_mx_batch(int32_t count, const float *const *srcs, const mqc_t4 *src_descs,
                                 const mqc_mx *mx, void *const *codes, uint8_t *const *scales,
                                 void *const *codes_alt, void *stream);

/* MX quantization with stochastic rounding of the elements (paper, section
 * III-A, Eq. 6 and the text after it: the gradients are rounded
 * stochastically, activations and weights to nearest).  Same arguments,
 * blocks, scales and layout as mqc_quantize_mx; only the element rounding
 * differs.  Each element x*2^-e lies between neighbouring magnitudes
 * lo <= |x*2^-e| < hi of the format; with f = (|x*2^-e| - lo) / (hi - lo)
 * and 16 random bits r, the magnitude is hi when r < f * 2^16, else lo
 * (hi with probability f to within 2^-16); values beyond the largest finite
 * magnitude saturate; the sign is kept.
 *   seed, offset  the random bits of element (b, a) at spatial position pix
 *           are bits 16*(j%4) .. 16*(j%4)+15 of word j/4 of the Philox4x64-10
 *           block (Salmon et al., "Parallel random numbers: as easy as 1, 2,
 *           3", SC 2011) with key (seed, 0) and counter (i/16, offset, 0, 0),
 *           where i = (pix*d0 + b)*A16 + a, A16 = d1 rounded up to 16 and
 *           j = i % 16.  The same (seed, offset) gives the same codes;
 *           callers draw a new offset (or seed) per step.
 * Requires mx->order == MQC_ORDER_BA (codes_alt may add the AB copy, with the
 * same rounding decisions) and an NCHW-like source: element stride 1 along
 * d3, d3 along d2, 16-byte aligned planes; else MQC_ERR_UNSUPPORTED before
 * any launch.
 * Errors: as mqc_quantize_mx, and MQC_ERR_UNSUPPORTED. */
MQC_API mqc_status mqc_quantize_mx_sr(const float *src, const mqc_t4 *src_desc, const mqc_mx *mx,
                              void *codes, uint8_t *scales, void *codes_alt, uint64_t seed,
                              uint64_t offset, void *stream);

/* NVFP4 block modes: blocks of 16 along the A-axis, along the B-axis, or a
 * 16 x 16 square over (B, A). */
typedef enum { MQC_NV_A16 = 0, MQC_NV_B16 = 1, MQC_NV_SQ16 = 2 } mqc_nv_block;

/* NVFP4 quantization, the format of the paper's own experiments (section
 * III-A, Eq. 4-6):
 *   Eq. 4  T  = max|X| / (448 * 6)                      per tensor, fp32
 *   Eq. 5  Bs = CastE4M3( max|X_i| / (T * 6) )          per block of 16, round to nearest even
 *   Eq. 6  q  = Round( x / (Bs * T) )                   E2M1, nearest even, saturating
 * each step one IEEE fp32 operation in that order; a block (or tensor) whose
 * scale is 0 gets zero codes.  Two launches: max|X| over the tensor, then
 * the blocks.
 *   block   an mqc_nv_block value; order BA or AB (as mqc_mx.order).
 *   codes   E2M1 codes in the layout of mqc_codes_bytes with fmt MQC_E2M1.
 *   scales  one E4M3 byte per block, mqc_nvfp4_scales_bytes() bytes:
 *             A16 : scales[(pix*Bp + b)*nb16(Ap) + a/16]
 *             B16 : scales[(pix*nb16(Bp) + b/16)*Ap + a]
 *             SQ16: scales[(pix*nb16(Bp) + b/16)*nb16(Ap) + a/16]
 *           (Ap, Bp the padded extents of `order`, nb16(x) = ceil(x/16)).
 *   codes_alt  optional second code order (shares the scales).
 *   tscale  device buffer of 2 floats: tscale[0] receives T; tscale[1] is
 *           scratch (the tensor maximum).
 * The source's spatial positions must be contiguous (element stride 1 along
 * d3, d3 along d2), else MQC_ERR_UNSUPPORTED.
 * Errors: MQC_ERR_INVALID, MQC_ERR_ALIGNMENT, MQC_ERR_UNSUPPORTED, MQC_ERR_CUDA. */
MQC_API mqc_status mqc_quantize_nvfp4(const float *src, const mqc_t4 *src_desc, int32_t block, int32_t order,
                              void *codes, uint8_t *scales, void *codes_alt, float *tscale, void *stream);
MQC_API int64_t mqc_nvfp4_scales_bytes(int32_t block, int32_t order, int32_t d0, int32_t d1, int32_t d2,
                               int32_t d3);

/* Channel-batch-first im2col on quantized X (paper, section IV-A): the
 * explicit expansion X'_{Cin,N} of shape (Kh Kw Cin) x (Hout Wout N).  The
 * output is the quantized layout above for a tensor with spatial P x Q,
 * B-axis N and A-axis (r, s, c) of extent R*S*Ap (c fastest), same format,
 * block mode and order as the input; positions in the zero padding get code
 * +0 and blocks wholly in the padding get scale 0x00.  When the blocked axes
 * are multiples of 32 the result is bit-identical to quantizing the fp32
 * im2col expansion.  Sizes: mqc_codes_bytes(mx, N, R*S*Ap, P, Q) (B32:
 * scales per tap as in the source).  The GEMMs never call this.
 * Errors: MQC_ERR_INVALID, MQC_ERR_ALIGNMENT. */
MQC_API mqc_status mqc_im2col_cbf(const void *codes, const uint8_t *scales, const mqc_conv *conv,
                          const mqc_mx *mx, void *codes_out, uint8_t *scales_out, void *stream);
MQC_API int64_t mqc_im2col_cbf_scales_bytes(const mqc_conv *conv, const mqc_mx *mx);
MQC_API int64_t mqc_im2col_cbf_codes_bytes(const mqc_conv *conv, const mqc_mx *mx);

/* The three GEMMs below take E4M3, E5M2 or E2M1 operands, in any mix.
 * Accumulation is fp32 in tensor memory (tcgen05.mma kind::mxf8f6f4 with
 * E8M0 block scales).  An E2M1 operand is first rewritten, in the caller's
 * workspace, as the E4M3 codes of the same values (every E2M1 value is an
 * E4M3 value; same layout, one byte per element); the products and the
 * scales are unchanged.  Each GEMM has a *_workspace_bytes query: 0 when no
 * operand is E2M1 (and, for the input gradient, the sub-pixel plan does not
 * apply; for the weight gradient, no split-K partials are needed), in which
 * case workspace may be NULL.  The workspace must be
 * 16-byte aligned; it is scratch, overwritten by the call.
 *
 * Forward convolution, Eq. 1, as the block-scaled GEMM
 * Y_f{Cout,N} = W_f{Cout,Cin} . X'_{Cin,N} of section IV-B, with the im2col
 * folded into the tensor-core operand staging.
 *   xq, xs  X quantized with blocks along C: block A32 or SQ32, order BA.
 *   wq, ws  W quantized with blocks along C: block A32 or SQ32, order BA.
 *   y       fp32 output [N][K][P][Q] (overwritten).
 *   workspace, workspace_bytes: at least mqc_conv2d_fwd_workspace_bytes().
 * Limits: R*S <= 64 kernel taps and stride_h*stride_w <= 4 (one activation
 * tensor map per stride phase); otherwise MQC_ERR_UNSUPPORTED before any
 * launch.
 * Errors: MQC_ERR_INVALID, MQC_ERR_UNSUPPORTED, MQC_ERR_ALIGNMENT, MQC_ERR_CUDA,
 * MQC_ERR_WORKSPACE. */
MQC_API mqc_status mqc_conv2d_fwd(const void *xq, const uint8_t *xs, const mqc_mx *xf,
                          const void *wq, const uint8_t *ws, const mqc_mx *wf,
                          const mqc_conv *conv, float *y,
                          void *workspace, size_t workspace_bytes, void *stream);
MQC_API size_t mqc_conv2d_fwd_workspace_bytes(const mqc_conv *conv, const mqc_mx *xf, const mqc_mx *wf);

/* Activations the quantized forward output can apply before quantizing. */
typedef enum { MQC_ACT_NONE = 0, MQC_ACT_RELU = 1, MQC_ACT_SILU = 2 } mqc_act;

/* Forward convolution whose output leaves the GEMM already quantized as the
 * next layer's input (the paper's flow of section V and Fig. 4: the
 * activation computed by a layer is on-chip, is quantized there and only the
 * quantized tensor is stored).  Same GEMM and operand requirements as
 * mqc_conv2d_fwd; the epilogue applies `act` to the fp32 accumulators
 * (MQC_ACT_RELU: max(x, 0); MQC_ACT_SILU: x / (1 + exp(-x)) in fp32), then
 * MX-quantizes the result Y [N][K][P][Q] as a tensor with B-axis N, A-axis
 * K and spatial P x Q, exactly as mqc_quantize_mx would quantize that fp32
 * tensor (round-to-nearest-even, same scale rule and layout).
 *   yf      format (E4M3, E5M2 or E2M1), block (A32 or SQ32) and order (BA).
 *   yq, ys  codes and scales: mqc_codes_bytes / mqc_scales_bytes of yf with
 *           dims (N, K, P, Q).
 *   yq_alt  optional (NULL): the same codes in order AB (the weight
 *           gradient's operand order), as mqc_quantize_mx's codes_alt.
 *   y       optional (NULL): an fp32 copy [N][K][P][Q] of the activated
 *           output that was quantized (for checking; the point of this call
 *           is not to write it).
 *   act     an mqc_act value.
 * Errors: as mqc_conv2d_fwd; MQC_ERR_UNSUPPORTED for order AB or B32. */
MQC_API mqc_status mqc_conv2d_fwd_quant(const void *xq, const uint8_t *xs, const mqc_mx *xf,
                                const void *wq, const uint8_t *ws, const mqc_mx *wf,
                                const mqc_conv *conv, int32_t act, const mqc_mx *yf, void *yq,
                                uint8_t *ys, void *yq_alt, float *y, void *workspace,
                                size_t workspace_bytes, void *stream);

/* Forward convolution (Eq. 1) with NVFP4 operands (the format of the paper's
 * experiments, section III-A, Eq. 4-7): the packed E2M1 codes go to the
 * tensor core as they are (tcgen05.mma kind::mxf4nvf4, K = 64 per
 * instruction, one UE4M3 scale per 16 elements of K, scale_vec::4X), and the
 * fp32 accumulators are multiplied by the two per-tensor scales T_x * T_w
 * (read on the device).
 *   xq, xs, x_tscale, x_block  X from mqc_quantize_nvfp4: order BA, block
 *           MQC_NV_A16 or MQC_NV_SQ16 (blocks along C), tscale[0] = T_x.
 *   wq, ws, w_tscale, w_block  W likewise (order BA, blocks along C).
 *   y       fp32 output [N][K][P][Q] (overwritten).
 * No workspace.  Limits as mqc_conv2d_fwd.
 * Errors: MQC_ERR_INVALID, MQC_ERR_UNSUPPORTED, MQC_ERR_ALIGNMENT, MQC_ERR_CUDA. */
MQC_API mqc_status mqc_conv2d_fwd_nvfp4(const void *xq, const uint8_t *xs, const float *x_tscale, int32_t x_block,
                                const void *wq, const uint8_t *ws, const float *w_tscale, int32_t w_block,
                                const mqc_conv *conv, float *y, void *stream);

/* Input gradient, Eq. 2: G_X = W^T * G_Y as the GEMM
 * G_X'{Cin,N} = W_f^T . G_Yf{Cout,N} of section IV-B, computed directly as a
 * transposed convolution; no G_X' is materialized.  When the stride phases
 * number 2 to 4, H and W are multiples of the strides and C is a multiple of
 * 16: ONE sub-pixel GEMM whose rows are the super-pixels (n, i, j) (input
 * pixels sh*i+ah, sw*j+aw for every phase (ah, aw)) and whose columns are
 * (phase, c), reducing over the few G_Y pixels (i+dh, j+dw) any phase
 * reaches; its weights (W's codes and scales rearranged per (dh, dw), zero
 * where no kernel tap links an offset to a phase) are built in the workspace
 * first, and the results are stored depth-to-space.  Otherwise one implicit
 * GEMM per output stride phase, up to four phases per kernel launch, their
 * tiles interleaved so that the phases' outputs (which interleave in memory)
 * are written together.  R*S <= 64; stride_h and stride_w at most 64.
 *   wq, ws  W quantized with blocks along K: block B32 or SQ32, order AB.
 *   gq, gs  G_Y quantized with blocks along K: block A32 or SQ32, order BA.
 *   gx      fp32 output [N][C][H][W] (overwritten).
 *   workspace, workspace_bytes: at least mqc_conv2d_bwd_data_workspace_bytes().
 * Errors: as mqc_conv2d_fwd. */
MQC_API mqc_status mqc_conv2d_bwd_data(const void *wq, const uint8_t *ws, const mqc_mx *wf,
                               const void *gq, const uint8_t *gs, const mqc_mx *gf,
                               const mqc_conv *conv, float *gx,
                               void *workspace, size_t workspace_bytes, void *stream);
MQC_API size_t mqc_conv2d_bwd_data_workspace_bytes(const mqc_conv *conv, const mqc_mx *wf, const mqc_mx *gf);

/* Weight gradient, Eq. 3: G_W[k,c] = sum_n G_Y[n,k] * X[n,c] as the GEMM
 * G_Wf{Cout,Cin} = G_Yf{Cout,N} . X'^T_{Cin,N} of section IV-B, reducing over
 * (Hout Wout N) with N contiguous (batch-first blocks).
 *   gq, gs  G_Y quantized with blocks along N: block B32 or SQ32, order AB.
 *   xq, xs  X quantized with blocks along N: block B32 or SQ32, order AB.
 *   gw      fp32 output [K][C][R][S] (overwritten).
 *   workspace, workspace_bytes: device scratch for the split-K partial sums
 *           and widened E2M1 operands, at least
 *           mqc_conv2d_bwd_weight_workspace_bytes(); may be NULL when that
 *           size is 0.
 * The split-K reduction is deterministic (fixed order).
 * Limits: R*S <= 64 and stride_h*stride_w <= 4, as mqc_conv2d_fwd.
 * Errors: as mqc_conv2d_fwd. */
MQC_API mqc_status mqc_conv2d_bwd_weight(const void *gq, const uint8_t *gs, const mqc_mx *gf,
                                 const void *xq, const uint8_t *xs, const mqc_mx *xf,
                                 const mqc_conv *conv, float *gw,
                                 void *workspace, size_t workspace_bytes, void *stream);
MQC_API size_t mqc_conv2d_bwd_weight_workspace_bytes(const mqc_conv *conv, const mqc_mx *gf, const mqc_mx *xf);

/* Size of the library's own split-K scratch array used by
 * mqc_conv2d_bwd_weight_noalloc (16 MiB, held on every GPU that loads the
 * library until the process exits). */
#define MQC_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/* Weight gradient that allocates nothing and takes no workspace.  (The paper
 * has no counterpart: this is a deployment convenience of this library.)
 * Same arguments, operand requirements and result as mqc_conv2d_bwd_weight,
 * but the split-K partial sums go to a fixed array inside the library
 * instead of caller memory.  It is meant for callers that cannot call
 * cudaMalloc or hand out scratch at the call site: plugin hosts whose device
 * memory is owned by someone else and frozen after start-up, and
 * latency-critical loops that cannot afford an allocation (and the device
 * synchronization cudaMalloc may imply) per call.
 *   - The first call on each device looks up that device's copy of the array
 *     (with the device current) and caches its address; make that first call
 *     before any stream capture.
 *   - A problem whose scratch (mqc_conv2d_bwd_weight_workspace_bytes: split-K
 *     partials and widened E2M1 operands) exceeds MQC_NOALLOC_SCRATCH_BYTES
 *     is rejected with MQC_ERR_WORKSPACE and nothing is launched.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's partial sums; each call overwrites every partial it later reads,
 *     so nothing needs to start at zero.  Calls that can overlap on the GPU
 *     (different streams, or different host threads) race on the array and
 *     must be serialized by the caller.
 * Errors: as mqc_conv2d_bwd_weight. */
MQC_API mqc_status mqc_conv2d_bwd_weight_noalloc(const void *gq, const uint8_t *gs, const mqc_mx *gf,
                                         const void *xq, const uint8_t *xs, const mqc_mx *xf,
                                         const mqc_conv *conv, float *gw, void *stream);

/* Synchronizes `stream`, then reads and clears the device error flag set by a
 * bounded wait that ran out.  MQC_OK if none; MQC_ERR_DEVICE_TIMEOUT if one
 * did; MQC_ERR_CUDA if the synchronization itself failed. */
MQC_API mqc_status mqc_get_device_status(void *stream);

/* Diagnostic: launches one thread that waits on a barrier nothing signals,
 * with a limit of `limit_ns` nanoseconds (1e3 .. 1e10), so that the bounded
 * wait runs out and sets the device error flag.  Lets a test exercise the
 * timeout path without hanging or faulting the GPU. */
MQC_API mqc_status mqc_debug_expire_wait(int64_t limit_ns, void *stream);

/* Static description of a status code; per-thread text of the last failure. */
MQC_API const char *mqc_status_string(mqc_status s);
MQC_API const char *mqc_last_error_message(void);

/* 100 * major + minor of this ABI. */
MQC_API int32_t mqc_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MQC_H */
