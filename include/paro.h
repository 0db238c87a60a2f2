/*
 * paro.h — C ABI of the B200 (sm_100a) library for ParoQuant's packed-inference
 * hot path: the scaled, pairwise-rotated INT4 linear layer.
 *
 * What the layer computes (GPTQModel wiki page "ParoQuant"):
 *   1. x <- x * channel_scales, per input channel; channel_scales is the saved
 *      runtime multiplier D^-1 (section "Activation and weight transforms").
 *   2. krot stages, in order, of disjoint Givens pair rotations inside every
 *      group of G input channels.  For a pair (a, b) with angle t:
 *          a' = a cos t + b sin t,   b' = -a sin t + b cos t
 *      (section "Pairwise Givens rotations").  Pair indices are local to the
 *      group; dummy pairs carry t = 0.
 *   3. Y = X_r . Q(W_r)^T + b against AWQ-packed int4 weights with group-wise
 *      scales and zero points (sections "Activation and weight transforms",
 *      "Stored tensors", "Triton plans and tuning": unpack INT4, subtract the
 *      zero point, multiply by the group scale, accumulate in fp32).
 *
 * Tensor layouts (section "Stored tensors"; I = K = in_features,
 * O = N = out_features, G = group size, all row-major, all little-endian):
 *   x, x_r          fp16    [M, K]   (bf16 through the *_dt entry points)
 *   channel_scales  fp32    [K]              (may be NULL: all ones)
 *   pairs           int16   [krot, K]        pairs[s, g*G+2p], pairs[s, g*G+2p+1]
 *                                            are the local channels (a, b) of pair p
 *                                            of stage s in group g, each in 0..G-1
 *   theta           fp32    [krot, K/2]      theta[s, g*G/2+p] is the angle of that pair
 *   qweight         int32   [K, N/8]         AWQ layout: nibble t (bits 4t..4t+3) of
 *                                            word w in row k holds column 8w+ORDER[t],
 *                                            ORDER = {0,2,4,6,1,3,5,7}
 *   qzeros          int32   [K/G, N/8]       same packing, 4-bit zero points
 *   scales          fp16    [K/G, N]         (same type as x)
 *   bias            fp16    [N]              (may be NULL; same type as x)
 *   y               fp16    [M, N]           (same type as x)
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, except the
 *     host-side helper paro_validate_pairs.  The library allocates nothing;
 *     scratch memory is a caller-provided workspace sized by the query function.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream) and
 *     return once the work is enqueued.  Inputs are never modified (except
 *     x in paro_rotate when x_r == x).  Outputs must not alias inputs otherwise.
 *   - Return value: PARO_OK, or a status found on the host before any launch
 *     (invalid shape or pointer, unsupported configuration, misalignment, small
 *     workspace), or PARO_ERR_CUDA if a launch failed.  Nothing is thrown or
 *     aborted across the ABI and nothing falls back to the CPU.
 *   - Kernels that wait on an mbarrier bound the wait; a wait that runs out sets
 *     a device status word that paro_device_status() reports as PARO_ERR_TIMEOUT.
 *   - Launch overlap.  paro_rotate and paro_w4_linear launch with programmatic
 *     dependent launch: a call's kernels may start while the kernel ahead of them
 *     in the stream is still running, and they read the layer constants
 *     (qweight, qzeros, scales, channel_scales, pairs, theta) before waiting for
 *     it; activations are read, and outputs and the workspace written, only
 *     after it has completed.  So the layer constants must not be written by the
 *     kernel immediately ahead of the call if that kernel releases its dependents
 *     early (griddepcontrol.launch_dependents).  No kernel of this library that
 *     releases early writes layer constants (paro_pack_awq does not release
 *     early; paro_quantize_w4 does not release early), and kernels that never
 *     release early are always safe.
 *   - Supported now: G in {16, 32, 64, 128} (the page's "Backend reference"
 *     lists groups 16/32/64/128 and -1; group_size == -1 is accepted when it
 *     normalises to one of these, i.e. K == 128, since K must be a multiple of
 *     128: the kernels work on 128-channel tiles holding 128 / G groups), the
 *     rotation groups and the quantisation groups share G; 0 <= krot <= 64;
 *     N a multiple of 32 (the packer alone needs only N % 8 == 0 and any even
 *     G); fp16 or bf16 activations/scales/bias/outputs (one type per call).
 *   - Activation type.  The plain entry points take fp16.  Each has a *_dt twin
 *     with one more argument, `dtype` (a paro_dtype), that selects fp16 or bf16
 *     for every 16-bit floating-point tensor of the call (x, x_r, w, scales,
 *     bias, y); any other value returns PARO_ERR_INVALID_ARG.  The page's
 *     "Stored tensors" section fixes no activation type (fp16 is the common
 *     serving type); the arithmetic is the same for both, only the final
 *     roundings and the tensor-core operand type change: in bf16 the weights
 *     (q - z) are still exact and products are still summed in fp32.
 */
#ifndef PARO_H_
#define PARO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* paro_stream_t;

typedef enum {
  PARO_OK = 0,
  PARO_ERR_INVALID_ARG = 1,  /* NULL pointer where data is needed, negative size, bad shape */
  PARO_ERR_UNSUPPORTED = 2,  /* valid per the method but not implemented (G not in {16,32,64,128}, ...) */
  PARO_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned (4-byte for fp32/int16 tables) */
  PARO_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than paro_w4_linear_workspace_size */
  PARO_ERR_CUDA = 5,         /* a CUDA launch or query failed */
  PARO_ERR_TIMEOUT = 6       /* a device-side wait ran out (see paro_device_status) */
} paro_status;

/* Type of the 16-bit floating-point tensors of a *_dt call. */
typedef enum {
  PARO_DTYPE_F16 = 0,   /* IEEE binary16 */
  PARO_DTYPE_BF16 = 1   /* bfloat16 */
} paro_dtype;

/* Static, NUL-terminated description of a status code (never NULL). */
const char* paro_status_string(int status);

/* Library version as "major.minor.patch". */
const char* paro_version(void);

/*
 * paro_rotate — X_r = rotate(x * channel_scales).
 * Defined by the page's "Pairwise Givens rotations" (pair formula, stage order,
 * group-local indices) and "Activation and weight transforms" (X_r = X D^-1 R).
 *   x, x_r          device fp16 [M, K], 16-byte aligned; x_r may equal x (in place)
 *   M >= 0 rows (M == 0 is a no-op), K > 0 channels, K % group_size == 0
 *   channel_scales  device fp32 [K] or NULL (no scaling)
 *   pairs, theta    device tables as above; may be NULL only when krot == 0
 *   group_size      16, 32, 64 or 128, or -1 meaning K (then K must be 128)
 *   krot            number of stages, 0..64 (0 = scaling only)
 * Arithmetic: fp32 on chip; cos/sin of the fp32 angle by the hardware
 * approximation after one reduction into [-pi, pi] (absolute error about
 * 2^-21); one round-to-nearest to fp16 (bf16) at the end.  Pair indices outside
 * 0..G-1 are masked into 0..G-1 (so no access leaves the group) and flagged in
 * the device status word; pair tables are not otherwise checked (see
 * paro_validate_pairs).
 */
int paro_rotate(const void* x, void* x_r, int64_t M, int64_t K, const float* channel_scales,
                const int16_t* pairs, const float* theta, int group_size, int krot,
                paro_stream_t stream);
int paro_rotate_dt(const void* x, void* x_r, int64_t M, int64_t K, const float* channel_scales,
                   const int16_t* pairs, const float* theta, int group_size, int krot, int dtype,
                   paro_stream_t stream);

/*
 * paro_rotate_rmat — X_r = rotate(x * channel_scales) as the product x R' with a
 * prepared R' (paro_rotation_matrix_prepare, which holds the channel scales,
 * pairs, theta, group size and krot), on the tensor cores: X R_hi + X R_lo
 * accumulated in fp32, rounded once to the activation type.  Any M (tiles
 * of 128 rows); the same result as paro_w4_linear's rotation above 64 rows.
 *   x, x_r   device [M, K] of `dtype`, 16-byte aligned, not the same buffer
 *   rmat     the prepared parts for this K and dtype, 256-byte aligned
 * Faster than paro_rotate for large M (the stages cost no more with krot).
 */
int paro_rotate_rmat(const void* x, void* x_r, int64_t M, int64_t K, const void* rmat, int dtype,
                     paro_stream_t stream);

/*
 * paro_pack_awq — pack 4-bit codes into AWQ int32 words (page "ParoQuant",
 * "Stored tensors": qweight (I, O//8), qzeros (I//G, O//8); packer needs O % 8 == 0).
 *   codes       device uint8 [N, K]    (out x in), values 0..15 (the high nibble is ignored)
 *   zero_codes  device uint8 [N, K/G]  values 0..15 (high nibble ignored); may be NULL
 *               together with qzeros == NULL to pack weights only
 *   qweight     device int32 [K, N/8]; qzeros device int32 [K/G, N/8]
 *   N % 8 == 0, K % G == 0, G even (any even G and any K is accepted here)
 * Bit-exact; the inverse is paro_unpack_awq.
 */
int paro_pack_awq(const uint8_t* codes, const uint8_t* zero_codes, int32_t* qweight,
                  int32_t* qzeros, int64_t N, int64_t K, int group_size, paro_stream_t stream);

/*
 * paro_quantize_w4 — packed runtime weights from float weights: the weight-side
 * transform W_r = W D R (page "ParoQuant", "Activation and weight transforms":
 * D = 1 / channel_scales, the rows of W taking the activations' stages) followed
 * by the four-bit symmetric quantiser of the same section (signed codes -8..7,
 * exported unsigned with zero point 8, quantiser scales bounded to [1e-5, 1e5])
 * and AWQ packing, in one pass.
 *   w               device fp16 [N, K] (out x in), 16-byte aligned
 *   channel_scales  device fp32 [K] (the runtime D^-1) or NULL (D = 1)
 *   pairs, theta    the layer's rotation tables (as for paro_rotate); NULL only when krot == 0
 *   scales          device fp16 [K/G, N] quantiser (= dequantisation) scales
 *   qweight         device int32 [K, N/8]; qzeros device int32 [K/G, N/8] (all 0x88888888)
 *   N >= 0, N % 8 == 0 (N == 0 is a no-op); K % 128 == 0; group_size 16, 32, 64 or 128 (or -1 with K == 128);
 *   krot 0..64; N * K < 2^31
 * Arithmetic: W * D with D = 1/channel_scales in fp32, the stages as in
 * paro_rotate (fp32, no fp16 rounding of W_r), q = rint(W_r * (1/s)) with ties
 * to even, s bounded first, then clamped to -8..7 and offset by 8.  A code can
 * differ from the exactly computed one only where W_r / s lies within the fp32
 * rounding of the transform of a half-integer.  Pair indices outside the group
 * are masked and flagged as in paro_rotate.  The kernel does not release its
 * dependents early, so a paro_w4_linear right after it may use its outputs.
 */
int paro_quantize_w4(const void* w, const float* channel_scales, const int16_t* pairs,
                     const float* theta, const void* scales, int32_t* qweight, int32_t* qzeros,
                     int64_t N, int64_t K, int group_size, int krot, paro_stream_t stream);
/* The same with w and scales of type `dtype` (the codes depend only on the
 * values of w and scales, read exactly in either type). */
int paro_quantize_w4_dt(const void* w, const float* channel_scales, const int16_t* pairs,
                        const float* theta, const void* scales, int32_t* qweight, int32_t* qzeros,
                        int64_t N, int64_t K, int group_size, int krot, int dtype, paro_stream_t stream);

/*
 * paro_quantize_w4_tc — paro_quantize_w4 on the tensor cores (fp16 weights).
 * The weight-side stages with D = 1 / channel_scales are one 128 x 128 map per
 * group, R'' = diag(D) G_0 ... G_{krot-1} (the product form of the page's
 * "Pairwise Givens rotations"); the call builds it into the workspace (two
 * fp16 parts, about 2^-22 relative), computes W_r = W R'' with tensor-core
 * MMAs into fp32 accumulators, and quantises and packs straight from them
 * (same quantiser, same words as paro_quantize_w4).
 *   Arguments as for paro_quantize_w4, plus N % 32 == 0 and a workspace of at
 *   least paro_quantize_w4_workspace_size(K) = K * 128 * 4 bytes, 256-byte
 *   aligned (contents need no initialisation).
 * W_r differs from paro_quantize_w4's fp32 stage-by-stage W_r by summation
 * order only (within a few units of 2^-22 of the group norm), so a code can
 * differ between the two only where W_r / s lies that close to a rounding
 * boundary.  Its last kernel does not release its dependents early.
 */
size_t paro_quantize_w4_workspace_size(int64_t K);
int paro_quantize_w4_tc(const void* w, const float* channel_scales, const int16_t* pairs,
                        const float* theta, const void* scales, int32_t* qweight, int32_t* qzeros,
                        int64_t N, int64_t K, int group_size, int krot, void* workspace,
                        size_t workspace_bytes, paro_stream_t stream);

/* paro_unpack_awq — exact inverse of paro_pack_awq (same shapes, same rules). */
int paro_unpack_awq(const int32_t* qweight, const int32_t* qzeros, uint8_t* codes,
                    uint8_t* zero_codes, int64_t N, int64_t K, int group_size,
                    paro_stream_t stream);

/*
 * paro_w4_linear_workspace_size — bytes of device workspace paro_w4_linear
 * needs for this shape (0 is possible).  Depends only on (M, K, N, group_size).
 * Returns 0 for shapes paro_w4_linear would reject.
 */
size_t paro_w4_linear_workspace_size(int64_t M, int64_t K, int64_t N, int group_size);

/*
 * paro_w4_linear — Y[M, N] = rotate(x * channel_scales) . dequant(qweight, qzeros, scales) + bias
 * with dequant(q, z, s)[k, n] = (q[k, n] - z[k/G, n]) * s[k/G, n]
 * (page "ParoQuant": "Activation and weight transforms" Y = X_r Q(W_r)^T + b;
 * "Triton plans and tuning" for the group-wise dequantisation with fp32 accumulation).
 *   krot == 0 skips the stages (pairs/theta ignored); channel_scales == NULL skips the
 *   scaling; both together give a plain AWQ W4 linear (the baseline of the
 *   rotation-overhead measurement).  bias may be NULL.
 *   x fp16 [M, K], y fp16 [M, N]: 16-byte aligned.  qweight, qzeros, scales:
 *   16-byte aligned.  workspace: device memory of at least
 *   paro_w4_linear_workspace_size(M, K, N, group_size) bytes, 256-byte aligned,
 *   contents need no initialisation and are clobbered; one workspace must not be
 *   used by two calls that can run at the same time.  After a call that rotates
 *   (krot > 0 or channel_scales != NULL) has completed, the first M*K*2 bytes of
 *   the workspace hold X_r (fp16 [M, K], row-major) until the workspace is used
 *   again; from M >= 65 the next 2*K*128*2 bytes hold the rotation matrices
 *   (below), the rest is scratch.
 *   Arithmetic: rotation in fp32 rounded once to fp16 (bf16); weights (q - z)
 *   exact in fp16 (bf16), times the group scale rounded to the activation type
 *   on the prefill path; products and sums in fp32 (tensor cores); y rounded
 *   once to fp16 (bf16).
 *   M <= 16 runs the decode GEMV path; larger M the tcgen05 prefill GEMM path.
 *   A prepared R' (paro_rotation_matrix_prepare, passed as paro_linear.rmat
 *   through paro_w4_linear_group, also with count == 1) replaces the per-call
 *   build above 64 rows.
 *   From M >= 65 the rotation itself runs on the tensor cores: each group's
 *   stages with its channel scales are the 128 x 128 matrix
 *   R' = diag(cs) G_0 ... G_{krot-1}, built per call in fp32 (its 128 basis rows
 *   taken through the stages) and stored as two parts of the activation type,
 *   R' = Rhi + Rlo; X_r = X Rhi + X Rlo accumulated in fp32 (R' kept to about
 *   2^-22 relative in fp16, about 2^-16 in bf16).
 *   Smaller batches apply the stages pair by pair.  paro_rotate always applies
 *   them pair by pair (it has no workspace for R').
 */
int paro_w4_linear(const void* x, void* y, int64_t M, int64_t K, int64_t N,
                   const int32_t* qweight, const int32_t* qzeros, const void* scales,
                   const void* bias, const float* channel_scales, const int16_t* pairs,
                   const float* theta, int group_size, int krot, void* workspace,
                   size_t workspace_bytes, paro_stream_t stream);
/* The same with x, scales, bias and y of type `dtype`; the workspace size does
 * not depend on the type. */
int paro_w4_linear_dt(const void* x, void* y, int64_t M, int64_t K, int64_t N,
                      const int32_t* qweight, const int32_t* qzeros, const void* scales,
                      const void* bias, const float* channel_scales, const int16_t* pairs,
                      const float* theta, int group_size, int krot, int dtype, void* workspace,
                      size_t workspace_bytes, paro_stream_t stream);

/*
 * Grouped decoder-layer calls — several linears that read the same x (a
 * decoder layer's q/k/v, or gate/up), each with its own weights, rotation
 * tables and output: y_i = rotate_i(x * cs_i) W_i + b_i for every member,
 * exactly as that many paro_w4_linear calls would compute it (page
 * "ParoQuant", "Activation and weight transforms": Y = X_r Q(W_r)^T + b per
 * member).  At decode sizes (M <= 16) the members share one rotation launch
 * and one GEMV launch when the combined grid is resident at once (for wide
 * members, gate and up, on a 2-stage ring with two CTAs per SM), else the
 * shared rotation launch is followed by one GEMV launch per member.  Above 16
 * rows one GEMM launch covers every member's column tiles.  Before it, above
 * 64 rows the rotating members share one R' build (skipped for members with a
 * prepared R') and one X R' launch; from 17 to 64 rows each distinct rotation
 * is one launch.  Members whose rotation
 * is the same — equal krot and the same channel_scales, pairs and theta
 * pointers (experts that share one rotation) — rotate x once: the first of
 * them computes X_r and the others read it.  Results may differ from the
 * separate calls in fp32 summation order only.
 *   linears         HOST array of `count` (1..PARO_MAX_GROUP) member descriptors;
 *                   each member's fields follow paro_w4_linear's rules
 *   x               device fp16 (or `dtype`) [M, K] shared by all members
 *   workspace       >= paro_w4_linear_group_workspace_size(...) bytes, 256-byte
 *                   aligned (may be NULL when no member rotates)
 */
#define PARO_MAX_GROUP 4
typedef struct paro_linear {
  int64_t N;                       /* output features of this member */
  const int32_t* qweight;          /* [K, N/8] */
  const int32_t* qzeros;           /* [K/G, N/8] */
  const void* scales;              /* fp16 (or dtype) [K/G, N] */
  const void* bias;                /* fp16 (or dtype) [N] or NULL */
  const float* channel_scales;     /* [K] or NULL */
  const int16_t* pairs;            /* [krot, K]; NULL only when krot == 0 */
  const float* theta;              /* [krot, K/2]; NULL only when krot == 0 */
  int krot;
  void* y;                         /* fp16 (or dtype) [M, N] output */
  /* Optional prepared R' parts of this member (paro_rotation_matrix_prepare
   * with this member's channel_scales, pairs, theta, K, group_size and krot,
   * in the call's dtype), 256-byte aligned, or NULL.  Batches above 64 rows
   * then skip the per-call R' build; nothing else changes (the same build
   * kernel made them, so results are identical). */
  const void* rmat;
} paro_linear;

size_t paro_w4_linear_group_workspace_size(int64_t M, int64_t K, int count, const paro_linear* linears,
                                           int group_size);
int paro_w4_linear_group(const void* x, int64_t M, int64_t K, int count, const paro_linear* linears,
                         int group_size, void* workspace, size_t workspace_bytes, paro_stream_t stream);
int paro_w4_linear_group_dt(const void* x, int64_t M, int64_t K, int count, const paro_linear* linears,
                            int group_size, int dtype, void* workspace, size_t workspace_bytes,
                            paro_stream_t stream);
/* Kernel launches paro_w4_linear_group issues for this group (rotations plus
 * GEMV/GEMM launches; 0 for an invalid shape or M == 0).  Host-only query; it
 * reads the current device's SM count and shared memory (cached per
 * device): whether decode members share one GEMV launch depends on whether
 * their grid is resident at once.  Without a device it counts one GEMV launch
 * per decode member. */
int paro_w4_linear_group_launches(int64_t M, int64_t K, int count, const paro_linear* linears,
                                  int group_size);

/*
 * paro_rotation_matrix_prepare — the R' parts of one layer, built once.
 * R' = diag(cs) G_0 ... G_{krot-1} per 128-channel tile (the product form of
 * the page's "Pairwise Givens rotations" with the channel scales of
 * "Activation and weight transforms") depends only on the stored rotation
 * (section "Stored tensors": channel_scales, pairs, theta), so a caller may
 * build it at load time and pass it with every call (paro_linear.rmat);
 * calls above 64 rows then skip their per-call build.
 *   channel_scales, pairs, theta, K, group_size, krot: as for paro_rotate
 *           (NULL pairs/theta only when krot == 0); K < 2^24
 *   dtype   the activation type of the calls that will use it (the parts are
 *           stored in that type: R' = Rhi + Rlo)
 *   rmat    device memory of at least paro_rotation_matrix_size(K) =
 *           K * 128 * 4 bytes, 256-byte aligned; written on `stream`
 * The build is the per-call one, so results do not change.  The kernel does
 * not release its dependents early, so a call right after may use rmat.
 * paro_rotation_matrix_size returns 0 for a K prepare would reject.
 */
size_t paro_rotation_matrix_size(int64_t K);
int paro_rotation_matrix_prepare(const float* channel_scales, const int16_t* pairs, const float* theta,
                                 int64_t K, int group_size, int krot, int dtype, void* rmat, size_t rmat_bytes,
                                 paro_stream_t stream);

/*
 * paro_w4_moe_linear — stacked experts that share one rotation: one
 * projection of a mixture-of-experts block (brain.gartu.xyz ParoQuant page,
 * MLX section: the experts' weights are stacked in one tensor and their
 * rotations are shared; each expert is the rotated W4 linear of the page
 * "ParoQuant", "Activation and weight transforms"):
 *   X_r = rotate(x * channel_scales)                   once, for every expert
 *   y[t, j, :] = X_r[t] . dequant(expert e) + bias[e],  e = expert_idx[t, j]
 *   x            device [T, K] (dtype), T >= 0 tokens (T == 0 is a no-op)
 *   expert_idx   device int32 [T, topk], 1 <= topk <= 64: the router's choice
 *                per token (any order; an expert may appear more than once)
 *   qweight      device int32 [E, K, N/8]; qzeros int32 [E, K/G, N/8];
 *   scales       [E, K/G, N] (dtype); bias [E, N] (dtype) or NULL;
 *                1 <= E <= 1024, each expert packed as for paro_w4_linear
 *   channel_scales, pairs, theta, krot: the one rotation of every expert
 *   y            device [T, topk, N] (dtype)
 *   workspace    >= paro_w4_moe_workspace_size(...) bytes, 256-byte aligned
 *   Shapes as for paro_w4_linear with M = T * topk (< 2^24); E * K < 2^31.
 * The call rotates x once, sorts the T * topk slots by expert on the device
 * (a stable counting sort: deterministic), copies each slot's X_r row into
 * the sorted order (in the sorting kernel itself when the routed rows take at
 * most 256 KB), then runs the decode GEMV over segments of at most 8
 * rows of one expert (T <= 16) or the tcgen05 GEMM over tiles of at most 256
 * rows of one expert, each writing its rows straight to their slots.  An
 * expert that no token selects costs nothing.  A slot whose index lies
 * outside 0..E-1 gets a zero row and is flagged in the device status word
 * (paro_device_status then reports PARO_ERR_INVALID_ARG).  Arithmetic as for
 * paro_w4_linear.  paro_w4_moe_launches is a host-only query of the kernel
 * launches one call issues (rotate != 0: the call rotates), 0 for a rejected
 * shape.
 */
size_t paro_w4_moe_workspace_size(int64_t T, int64_t K, int64_t N, int E, int topk, int group_size);
int paro_w4_moe_linear(const void* x, void* y, int64_t T, int64_t K, int64_t N, int E, int topk,
                       const int32_t* expert_idx, const int32_t* qweight, const int32_t* qzeros,
                       const void* scales, const void* bias, const float* channel_scales,
                       const int16_t* pairs, const float* theta, int group_size, int krot, int dtype,
                       void* workspace, size_t workspace_bytes, paro_stream_t stream);
int paro_w4_moe_launches(int64_t T, int64_t K, int64_t N, int E, int topk, int group_size, int krot,
                         int rotate);

/*
 * paro_w4_linear_noalloc — paro_w4_linear for callers that cannot allocate
 * device memory.  The paper has no counterpart; this entry point exists for
 * library users, not for the method.
 *
 * Some callers cannot hand this library a workspace: code that records CUDA
 * graphs in the global capture mode (cudaMalloc is not allowed there),
 * latency-critical loops that must not pay cudaMalloc's implicit device
 * synchronisation, and plugin hosts that own all device memory and forbid a
 * library from allocating outside their pool.  This variant takes the same
 * arguments as paro_w4_linear minus the workspace and stages X_r in a
 * file-scope device array of PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES bytes that
 * every GPU which loads the library holds until the process exits.  It calls
 * no cudaMalloc, cudaFree or allocating library routine.
 *   - Limit: a call that rotates (krot > 0 or channel_scales != NULL) needs
 *     paro_w4_linear_workspace_size(M, K, N, group_size) <=
 *     PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES (8 MiB: M*K <= 4 Mi fp16 elements
 *     up to 64 rows; above 64 rows M*K*2 + 512*K bytes, e.g. M <= 768 at
 *     K = 4096); larger shapes return PARO_ERR_WORKSPACE before any GPU work.
 *     A call that does not rotate stages nothing and has no limit.  Arguments
 *     are checked first, exactly as paro_w4_linear checks them, so a bad
 *     argument gets the same status from both entry points.
 *   - The first call on a device looks up the array's device address for that
 *     device (cudaGetSymbolAddress) and caches it; make that first call before
 *     any stream capture.
 *   - Every call shares the one array, which keeps the last call's contents (it
 *     needs no clearing: each call overwrites what it reads).  Calls whose work
 *     can overlap on the GPU (different streams, or different host threads on
 *     one device) race on the array; serialise them, or use paro_w4_linear with
 *     separate workspaces.
 * Results are those of paro_w4_linear for the same arguments.
 */
#define PARO_W4_LINEAR_NOALLOC_SCRATCH_BYTES (8u << 20)

int paro_w4_linear_noalloc(const void* x, void* y, int64_t M, int64_t K, int64_t N,
                           const int32_t* qweight, const int32_t* qzeros, const void* scales,
                           const void* bias, const float* channel_scales, const int16_t* pairs,
                           const float* theta, int group_size, int krot, paro_stream_t stream);
int paro_w4_linear_noalloc_dt(const void* x, void* y, int64_t M, int64_t K, int64_t N,
                              const int32_t* qweight, const int32_t* qzeros, const void* scales,
                              const void* bias, const float* channel_scales, const int16_t* pairs,
                              const float* theta, int group_size, int krot, int dtype, paro_stream_t stream);

/*
 * paro_validate_pairs — HOST helper (host pointer, synchronous, no GPU work):
 * checks that every stage of every group of a [krot, K] pair table is a
 * permutation of 0..G-1 (each channel in exactly one pair; cf. the page's
 * "validated local pair permutations").  Returns PARO_OK or PARO_ERR_INVALID_ARG.
 */
int paro_validate_pairs(const int16_t* pairs_host, int64_t K, int group_size, int krot);

/*
 * paro_device_status — reads (and, if clear != 0, resets) the device status word
 * of the current device.  Synchronises the device.  Returns PARO_OK,
 * PARO_ERR_TIMEOUT (a bounded wait ran out), PARO_ERR_INVALID_ARG (a pair index
 * outside its group, or an expert index outside 0..E-1, was seen) or
 * PARO_ERR_CUDA (the CUDA query failed).
 */
int paro_device_status(int clear);

/*
 * paro_selftest_wait_timeout — failure-detection self-test (the pages have no
 * counterpart; it checks this library's own error path).  Runs one kernel whose
 * single thread waits, with the bounded wait every kernel of this library uses
 * but a limit of `limit_ns` nanoseconds, on an mbarrier that nothing arrives
 * at.  The wait runs out, sets the timeout bit of the device status word (so
 * paro_device_status then reports PARO_ERR_TIMEOUT) and the kernel returns
 * normally; no copy or other work is in flight, and the context stays usable.
 *   limit_ns    1 .. 100 000 000 (100 ms), else PARO_ERR_INVALID_ARG
 *   elapsed_ns  HOST pointer or NULL: nanoseconds the wait took before giving up
 *               (device %globaltimer), 0 if it had completed instead
 * Synchronises `stream`.  Returns PARO_OK once the kernel has run, or
 * PARO_ERR_CUDA if the launch or the read-back failed.
 */
int paro_selftest_wait_timeout(uint64_t limit_ns, uint64_t* elapsed_ns, paro_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PARO_H_ */
