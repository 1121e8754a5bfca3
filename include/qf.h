/*
 * qf.h -- C ABI of the B200 (sm_100a) deployment-aligned simulated-quantization
 * library (libqf.so).
 *
 * The library implements the hot path of quantization-aware training as
 * described on the QATFactory project page ("QATFactory: A Versatile,
 * Deployment-Aligned Framework for Quantization-aware Training and Distillation
 * of LLMs"): in the forward pass every weight (and, if wanted, activation)
 * becomes the nearest value a deployment format can hold (quantize, then
 * dequantize); in the backward pass the gradient passes straight through to the
 * full-precision weight; and the codes and scales are written in the byte
 * layout the inference engine loads.
 *
 * Formats ("Supported formats" table of the project page):
 *   NVFP4  E2M1 elements, 16-element blocks, E4M3 block scale, FP32 tensor scale,
 *          symmetric, 4.50 bits/weight
 *   MXFP4  E2M1 elements, 32-element blocks, E8M0 block scale, symmetric,
 *          4.25 bits/weight
 *   Q4_K   unsigned 4-bit elements, 32-element sub-blocks in 256-element
 *          super-blocks, 6-bit sub-block scale and min, FP16 super-block d and
 *          dmin, asymmetric, 4.50 bits/weight
 *
 * Conventions common to every call
 *   - A tensor is a row-major, contiguous BF16 matrix [rows, cols].  Blocks run
 *     along cols (the contiguous dimension, the GEMM reduction dimension along
 *     which the engines scale); cols must be a multiple of the format's block
 *     (16, 32 or 256).  Since blocks never straddle rows, element i of the
 *     tensor (flat index) belongs to block i / block_size.
 *   - Every pointer in a qf_tensor and every d_* pointer is a DEVICE pointer on
 *     the current CUDA device, owned by the caller.  The library allocates no
 *     memory and keeps no pointer after a call returns.  The qf_tensor array
 *     itself is HOST memory, read during the call only.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call
 *     is asynchronous on that stream.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns an error status and launches nothing.  A CUDA launch
 *     failure returns QF_ERR_CUDA.  Kernels never trap.  The one wait on other
 *     threads in the library is the grid barrier of qf_amax_fakequant's
 *     single-launch path, which is bounded (see there).  The LoRA kernels also
 *     wait, in hardware (cp.async.wait_group), for their own asynchronous copies
 *     of W into shared memory.
 *     qf_last_error() gives a one-line description of the last failure on the
 *     calling thread.
 *   - Outputs must not overlap the inputs or one another, except that
 *     qf_ste_backward accepts grad_x == grad_y (mode 0 then launches nothing; mode 1
 *     reads the gradient with ordinary loads, each element before it is written).
 *     The kernels read x through the read-only (non-coherent) path.
 *   - Calls on the same stream are ordered; calls whose outputs overlap and that
 *     run concurrently on different streams race.
 *   - Numerics are fixed bit for bit (see each call); every result is
 *     deterministic and independent of launch configuration.
 */
#ifndef QF_H
#define QF_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QF_NVFP4 = 0,
    QF_MXFP4 = 1,
    QF_Q4K = 2,
    QF_Q4K_MSE = 3      /* Q4_K with the MSE-searched sub-block scales (same layout) */
} qf_format;

typedef enum {
    QF_OK = 0,
    QF_ERR_INVALID_ARG = 1,   /* null pointer, bad count, group out of range, no output */
    QF_ERR_SHAPE = 2,         /* negative or overflowing size, cols not a block multiple */
    QF_ERR_ALIGN = 3,         /* x / y / codes not 16-byte aligned */
    QF_ERR_UNSUPPORTED = 4,   /* unknown format or mode */
    QF_ERR_CUDA = 5,          /* a CUDA call failed (see qf_last_error) */
    QF_ERR_TIMEOUT = 6        /* a bounded device wait gave up (qf_workspace_check) */
} qf_status;

/* Element type of the input x (qf_tensor.x_type). */
#define QF_X_BF16 0             /* BF16 weights or activations */
#define QF_X_F32 1              /* FP32 latent (master) weights */

#define QF_NVFP4_BLOCK 16
#define QF_MXFP4_BLOCK 32
#define QF_Q4K_SUBBLOCK 32
#define QF_Q4K_SUPERBLOCK 256
#define QF_Q4K_BLOCK_BYTES 144

/*
 * One tensor of a call.
 *   x       [rows, cols] of x_type elements, 16-byte aligned.  May be NULL only if
 *           rows*cols == 0.
 *   rows    >= 0
 *   cols    >= 0, a multiple of the format's block size
 *   group   NVFP4 tie group in [0, n_groups): every tensor of a group shares one
 *           FP32 tensor scale (the projections an engine fuses, e.g. Q, K and V,
 *           or gate and up -- project page, Method, "Numerics").  Ignored by
 *           MXFP4 and Q4_K.
 *   x_type  QF_X_BF16 (0) or QF_X_F32 (1): BF16 inputs, or the FP32 latent weights a
 *           full-parameter training run keeps (the project page's memory table lists
 *           the student's trainable weights as FP32).  Every tensor of one call has
 *           the same x_type.  The outputs are the same for both: BF16 y, codes,
 *           scales; an FP32 element that is a BF16 value gives the BF16 result.
 *   y       BF16 [rows, cols] dequantized output, 16-byte aligned, or NULL
 *   codes   packed output, 16-byte aligned, or NULL:
 *             NVFP4 / MXFP4: rows*cols/2 bytes; element 2i of the flat tensor in
 *               bits 0-3 of byte i, element 2i+1 in bits 4-7; each nibble is an
 *               E2M1 code (bit 3 = sign).
 *             Q4_K: (rows*cols/256) blocks of 144 bytes, one per super-block in
 *               flat order: FP16 d, FP16 dmin, 12 bytes of 6-bit scales/mins,
 *               128 bytes of 4-bit codes (the GGUF Q4_K block layout).
 *   scales  block scales, any alignment, or NULL (ignored by Q4_K, whose scales
 *           live inside its blocks):
 *             NVFP4: rows*cols/16 E4M3 bytes, MXFP4: rows*cols/32 E8M0 bytes,
 *             row-major (flat block order).
 */
typedef struct qf_tensor {
    const void* x;
    int64_t rows;
    int64_t cols;
    int32_t group;
    int32_t x_type;
    void* y;
    void* codes;
    void* scales;
} qf_tensor;

/*
 * qf_amax_tied -- tied NVFP4 tensor amax (project page, Method, "Numerics": a
 * projection group that vLLM or SGLang runs as one fused GEMM uses a common
 * tensor scale; "Export": the NVFP4 activation amax is kept from training, so
 * serving needs no calibration).
 *
 *   d_group_amax[g] = max over the tensors i with t[i].group == g of max |x_i|
 *                     (FP32, exact); 0 for a group with no tensor.  Overwritten.
 *   d_tracked       NULL, or FP32[n_groups]: updated in place to
 *                     max(d_tracked[g], d_group_amax[g])  (the running amax a
 *                     training loop keeps for activations; pass it as the
 *                     d_group_amax of qf_fakequant to quantize with it).  Its
 *                     values must be >= +0 (start it at +0): the max is taken on
 *                     the FP32 bit patterns as unsigned integers, which is the
 *                     float max there (a NaN running value stays NaN).
 *   Only x, rows, cols, group and x_type of each tensor are read; cols may be any
 *   value >= 0 here.  n == 0 only clears d_group_amax.
 * Errors: t == NULL with n > 0, n < 0, n_groups <= 0, d_group_amax == NULL,
 *   group out of range -> QF_ERR_INVALID_ARG; bad sizes -> QF_ERR_SHAPE;
 *   x not 16-byte aligned -> QF_ERR_ALIGN.
 */
qf_status qf_amax_tied(const qf_tensor* t, int n, float* d_group_amax, int n_groups,
                       float* d_tracked, void* stream);

/*
 * qf_fakequant -- the fused forward pass: block statistics, block-scale encode,
 * element encode, dequantize and pack in one read of x (project page, Method,
 * "Framework overview": quantize then dequantize so training sees serving's
 * numbers; "QARL"/"Export": the engine's byte layout).  n == 1 is one
 * tensor; n > 1 is one grouped launch over all n tensors (e.g. every expert of
 * an MoE layer), bitwise identical to n single calls.
 *
 * Numerics (IEEE binary32, round to nearest even, no fused multiply-add):
 *   NVFP4: s_t = amax_g / 2688 (= amax_g / (6 * 448)), amax_g = d_group_amax[group];
 *          per 16-block: sb = E4M3_satfinite(amax_b / (6 * s_t)) (sb = 0 if s_t == 0),
 *          S = f32(sb) * s_t, inv = 1 / S (0 if S == 0),
 *          code = E2M1_satfinite(x * inv) (a zero x stays a zero of its sign),
 *          y = BF16(f32(code) * S).
 *   MXFP4: per 32-block: e = clamp(floor(log2 amax_b) - 2, -127, 127)
 *          (-127 for an all-zero block), scale byte = e + 127,
 *          code = E2M1_satfinite(x * 2^-e), y = BF16(f32(code) * 2^e).
 *   Q4_K:  per 32-sub-block j: min_j = max(-min x, 0), scale_j = (max x + min_j) / 15;
 *          d = FP16(max_j scale_j / 63), dmin = FP16(max_j min_j / 63);
 *          sc_j = min(RNE(scale_j / d), 63) (0 if d == 0), m_j likewise with dmin;
 *          s_j = d * sc_j, mm_j = dmin * m_j, inv_j = 1 / s_j (0 if s_j == 0);
 *          q = clamp(RNE((x + mm_j) * inv_j), 0, 15), y = BF16(s_j * q - mm_j).
 *   E2M1 codes carry the sign bit of their input (a negative value that rounds
 *   to zero gives code 8).
 *
 *   d_group_amax       NVFP4: FP32[n_groups] device array of tie-group amaxes
 *                      (from qf_amax_tied).  Ignored by MXFP4 / Q4_K (may be NULL).
 *   n_groups           NVFP4: number of entries of d_group_amax (> 0).
 *   d_group_scale_out  NVFP4: NULL, or FP32[n_groups] receiving each s_t.
 * Every tensor needs at least one of y, codes, scales non-NULL.
 * Errors: unknown format -> QF_ERR_UNSUPPORTED; see qf_tensor for the rest.
 */
qf_status qf_fakequant(qf_format f, const qf_tensor* t, int n, const float* d_group_amax,
                       int n_groups, float* d_group_scale_out, void* stream);

/*
 * qf_amax_fakequant -- NVFP4 tie-group amax and fused fake-quant + pack in one call:
 * the results of qf_amax_tied followed by qf_fakequant(QF_NVFP4, ...) on the
 * scale it gives, bit for bit.  The tensor scale needs the amax of the whole tie
 * group before any block is encoded (project page, Method, "Numerics": one FP32
 * tensor scale per fused projection group), which costs a second pass over x.
 *
 * When every input fits comfortably in L2 (all x bytes <= L2 size / 3: up to
 * about 44 MB on a B200), a workspace is given, n <= 384 and the device supports
 * cooperative launches, both passes run in ONE cooperative launch.  The first
 * pass reads x from HBM and folds max |x| into the workspace.  A grid-wide
 * barrier follows.  The second pass re-reads x from L2 and encodes it.
 * Otherwise, or with d_workspace == NULL, the call makes the two launches of
 * qf_amax_tied and qf_fakequant.
 *
 *   t, n, n_groups     as for qf_fakequant with QF_NVFP4 (every check of
 *                      qf_amax_tied and qf_fakequant is made before any launch).
 *   d_group_amax       FP32[n_groups], overwritten with this call's group amax.
 *   d_tracked          NULL, or FP32[n_groups] running amax, updated in place to
 *                      max(d_tracked[g], amax_g); when given, s_t is taken from
 *                      the updated running value (activations), otherwise from
 *                      amax_g (weights).
 *   d_group_scale_out  NULL, or FP32[n_groups] receiving each s_t.
 *   d_workspace        NULL, or device memory of at least
 *                      qf_amax_fakequant_workspace_bytes(n_groups) bytes,
 *                      16-byte aligned, ALL ZERO before its first use (e.g.
 *                      cudaMemset once).  Every call that completes leaves it zero
 *                      again, so it can be reused by later calls on the same stream.
 *                      Calls that may overlap (different streams) need their own
 *                      workspaces.
 *   workspace_bytes    its size.
 * The barrier wait is bounded (about a second of polling).  A CTA that gives up
 * sets an error flag in the workspace and writes none of its outputs; every CTA
 * still leaves the workspace's counters and slots zeroed.  The flag is sticky: until
 * qf_workspace_check reads and clears it, every later call on that workspace does no
 * work at all (its outputs are left as they were), so no call can encode from a
 * partial amax.  Check the workspace after any call whose outputs matter.  A
 * cooperative launch guarantees that every CTA is resident, so the wait completes
 * unless a CTA faults.
 * Amax folding: every max (the group amax, the running value) is taken on the FP32
 *   bit patterns as unsigned integers, as qf_amax_tied does; that is the float max for
 *   values >= +0, so the running amax must start at +0 (or any value >= +0).  A NaN in
 *   x or in d_tracked is outside the formats (inputs are finite), but both paths of
 *   this call give the same bytes for it (a NaN running value stays NaN).
 * Errors: as qf_fakequant; a workspace smaller than needed -> QF_ERR_INVALID_ARG,
 *   not 16-byte aligned -> QF_ERR_ALIGN.
 */
qf_status qf_amax_fakequant(const qf_tensor* t, int n, float* d_group_amax, int n_groups,
                            float* d_tracked, float* d_group_scale_out, void* d_workspace,
                            size_t workspace_bytes, void* stream);

/* Bytes of workspace qf_amax_fakequant needs for n_groups tie groups (0 if n_groups <= 0). */
size_t qf_amax_fakequant_workspace_bytes(int n_groups);

/*
 * qf_amax_fakequant_noalloc -- qf_amax_fakequant with a workspace the library owns:
 * a static device array of 16 KB per device, compiled into libqf.so.  No memory is
 * allocated, neither by this call nor by the caller.  The project page has no
 * counterpart: this is an interface convenience, not part of the method.
 *
 * The results are bit for bit those of qf_amax_fakequant with a caller workspace.
 * The call first clears the counters and slots of the static workspace (one
 * cudaMemsetAsync on `stream`), then runs qf_amax_fakequant on it.  Its error word is
 * not cleared: a barrier timeout stays recorded, and every later call does no work,
 * until qf_noalloc_check reads and clears it.
 * Limit: n_groups <= 4092; larger counts return QF_ERR_INVALID_ARG (use
 * qf_amax_fakequant with a workspace of your own).
 * The static workspace is shared by every call on the device.  Two calls that may
 * run at the same time (different streams, or different host threads with no
 * ordering between them) race on it: serialize them, or give each its own
 * workspace through qf_amax_fakequant.
 * Errors: as qf_amax_fakequant.
 */
qf_status qf_amax_fakequant_noalloc(const qf_tensor* t, int n, float* d_group_amax,
                                    int n_groups, float* d_tracked, float* d_group_scale_out,
                                    void* stream);

/* Synchronizes `stream`, then reads the error flags of a qf_amax_fakequant
 * workspace and clears them: QF_OK, or QF_ERR_TIMEOUT if a grid barrier gave up
 * (that call, and every later call on the workspace before this check, wrote no
 * outputs).  The workspace is ready for reuse either way. */
qf_status qf_workspace_check(const void* d_workspace, void* stream);

/* qf_workspace_check for the static workspace of qf_amax_fakequant_noalloc on the
 * current device. */
qf_status qf_noalloc_check(void* stream);

/* Testing aid for the timeout path of the single-launch grid barrier.  With polls > 0,
 * every later qf_amax_fakequant* call of this process that takes the single-launch
 * path waits for one CTA more than its grid holds, polls at most `polls` times
 * (about 256 ns apart), and gives up: the timeout is reported as above, with every
 * CTA present and nothing faulted.  polls == 0 (the default) restores normal
 * operation.  Not for production use. */
void qf_test_barrier_timeout(unsigned int polls);

/*
 * qf_pack -- the engine-layout export and weight sync (project page, Method,
 * "QARL": after every optimizer step the trainer writes its weights in the
 * engine's byte layout and hands them over; "Export").  Identical to qf_fakequant except that y is never
 * written (it may be non-NULL and is ignored); each tensor needs codes or scales.
 * The bytes written are those qf_fakequant writes.
 */
qf_status qf_pack(qf_format f, const qf_tensor* t, int n, const float* d_group_amax,
                  int n_groups, float* d_group_scale_out, void* stream);

/*
 * qf_ste_backward -- straight-through estimator backward (project page, Method,
 * "Framework overview": the gradient reaches the full-precision weights
 * unchanged by the rounding; Bengio,
 * Leonard and Courville 2013, cited by the paper).
 *   mode 0 (identity):  grad_x = grad_y, numel BF16 elements.  grad_x == grad_y
 *                       is allowed and launches nothing.  f, fwd and
 *                       d_group_amax are ignored.
 *   mode 1 (clipped):   grad_x = grad_y where the forward pass did not saturate
 *                       the element, +0 elsewhere: NVFP4/MXFP4 |x * inv| <= 6,
 *                       Q4_K 0 <= (x + mm_j) * inv_j <= 15, with the scales the
 *                       forward pass of format f derives for fwd->x.  fwd gives x,
 *                       x_type, rows, cols and (NVFP4) group; numel == rows * cols;
 *                       d_group_amax as for qf_fakequant (NVFP4 only).
 *   grad_y, grad_x: BF16 device arrays, 16-byte aligned.
 * Errors: mode not 0/1 or unknown format -> QF_ERR_UNSUPPORTED; the rest as above.
 */
qf_status qf_ste_backward(qf_format f, const void* grad_y, void* grad_x, int64_t numel,
                          int mode, const qf_tensor* fwd, const float* d_group_amax,
                          int n_groups, void* stream);

/*
 * LoRA adapters (project page, Method, "QAD": LoRA-QAD trains low-rank adapters
 * on a frozen BF16 base and quantizes the merged weight, not the base).
 * For tensor t with base W = t.x (BF16 [rows, cols]):
 *   acc = sum over k = 0..rank-1, in increasing k, of b[i,k] * a[k,j]   (FP32; each
 *         term is one fused multiply-add, acc + b*a rounded once)
 *   M   = BF16( W[i,j] + scale * acc )      (an FP32 multiply, an FP32 add, RNE)
 * M is the merged weight a BF16 model holds after merging the adapter.
 *   b       BF16 [rows, rank] row-major (device)
 *   a       BF16 [rank, cols] row-major (device), 16-byte aligned
 *   rank    1 .. QF_LORA_MAX_RANK
 *   scale   FP32 multiplier of B A (alpha / rank in the usual parameterisation)
 */
#define QF_LORA_MAX_RANK 32
typedef struct qf_lora {
    const void* b;
    const void* a;
    int32_t rank;
    float scale;
} qf_lora;

/*
 * qf_lora_merge -- writes the merged weight M of each tensor to t[i].y (BF16
 * [rows, cols]); codes and scales are ignored.  Use it to feed qf_fakequant with
 * formats qf_fakequant_lora does not fuse (Q4_K).
 * qf_amax_tied_lora -- qf_amax_tied of the merged weights (NVFP4 tie groups).
 * qf_fakequant_lora -- qf_fakequant of the merged weights, NVFP4 or MXFP4, with the
 *   merge formed on the fly (M is never written): bitwise the same outputs as
 *   qf_lora_merge followed by qf_fakequant.
 * All three: t[i].x_type must be QF_X_BF16; cols a multiple of 16 (MXFP4: 32);
 * l[i] is the adapter of t[i].  Errors as for the calls without LoRA, plus
 * QF_ERR_INVALID_ARG for a NULL adapter pointer or a rank outside
 * [1, QF_LORA_MAX_RANK], QF_ERR_UNSUPPORTED for FP32 bases or (qf_fakequant_lora)
 * the Q4_K format.
 */
qf_status qf_lora_merge(const qf_tensor* t, const qf_lora* l, int n, void* stream);
qf_status qf_amax_tied_lora(const qf_tensor* t, const qf_lora* l, int n, float* d_group_amax,
                            int n_groups, void* stream);
qf_status qf_fakequant_lora(qf_format f, const qf_tensor* t, const qf_lora* l, int n,
                            const float* d_group_amax, int n_groups, float* d_group_scale_out,
                            void* stream);

/*
 * qf_amax_fakequant_lora -- the LoRA-QAD NVFP4 step in one call: the tie-group amax
 * of the merged weights (as qf_amax_tied_lora), then their fake-quant + pack (as
 * qf_fakequant_lora with QF_NVFP4 on that amax).  The outputs are bit for bit those
 * of the two calls.
 *   When every non-empty tensor has a y, the merged weight is formed ONCE: one
 *   pass writes BF16(W + scale * B A) into y and folds its max |M| into the group
 *   amax, and the plain NVFP4 fused pass then quantizes y in place.  Otherwise the
 *   merge is formed in both passes, as the two calls do.
 *   t, l, n, n_groups   as for qf_fakequant_lora with QF_NVFP4.
 *   d_group_amax        FP32[n_groups], overwritten with the merged weights' group amax.
 *   d_group_scale_out   NULL, or FP32[n_groups] receiving each s_t.
 * Errors: as qf_amax_tied_lora and qf_fakequant_lora.
 */
qf_status qf_amax_fakequant_lora(const qf_tensor* t, const qf_lora* l, int n,
                                 float* d_group_amax, int n_groups, float* d_group_scale_out,
                                 void* stream);

/*
 * QF_Q4K_MSE -- the Q4_K format (identical 144-byte blocks and dequantization) with
 * an MSE-searched fit, the kind of post-training quantizer the project page uses as
 * its Q4_K PTQ baseline ("Key findings"; the pages do not give its steps).  Per
 * 32-element sub-block, with min_j as in the min/max fit, the scale is chosen among
 * (max x + min_j) / n for n = 15 (tried first), 14, 14.5, 15.5, 16, 16.5, 17, 17.5, 18
 * as the one with the least
 *   err = sum over i, in order, of (x_i - (scale*q_i - min_j))^2,
 *   q_i = clamp(RNE((x_i + min_j) * (1/scale)), 0, 15)
 * (binary32, one rounding per operation; a later n must be strictly better); then
 * d, dmin, sc, m and the codes follow exactly as for QF_Q4K.  Accepted by
 * qf_fakequant, qf_pack and qf_ste_backward.
 */

/* Static description of a status code. */
const char* qf_status_string(qf_status s);

/* One-line description of the last failed call on the calling thread ("" if none). */
const char* qf_last_error(void);

/* ABI version: (major << 16) | minor.  1.1 added qf_tensor.x_type (formerly a
 * reserved field that had to be 0, which still means BF16); 1.2 the LoRA calls;
 * 1.3 QF_Q4K_MSE; 1.4 qf_amax_fakequant, its workspace calls and QF_ERR_TIMEOUT;
 * 1.5 qf_amax_fakequant_noalloc; 1.6 qf_amax_fakequant_lora; 1.7 sticky workspace
 * error flags, qf_noalloc_check and qf_test_barrier_timeout. */
int qf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QF_H */
