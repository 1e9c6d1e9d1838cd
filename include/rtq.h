/*
 * rtq.h -- C ABI of the B200 weight-only quantized projection GEMM.
 *
 * The operation (both RT-J quantized model cards, opening paragraph): a
 * transformer-block projection Y[M,N] = X[M,K] * W[N,K]^T whose weights stay
 * quantized in device memory and are dequantized inside the GEMM, so the only
 * weight traffic is the quantized payload.  Two weight formats:
 *
 *   q4  ("RT-J -- int4 (Q4-style, mixed-precision) quantized checkpoints",
 *       section "Quantization format"): uint4 codes in groups of 32 along the
 *       input dimension K, packed two per byte with the LOW nibble holding the
 *       EVEN index; one fp16 (scale, min) pair per group;
 *       W[o,k] = code(o,k) * scale[o,k/32] + min[o,k/32].
 *         Wq        uint8  [N, K/2], row-major
 *         scale_min uint16 [N, K/32, 2], binary16 bits, element 0 = scale,
 *                   element 1 = min (the pages give a "(scale, min) pair per
 *                   group" in one companion tensor; the interleaved order is
 *                   this library's reading)
 *
 *   q8  ("RT-J -- int8 (Q8_0-style) quantized checkpoints", section
 *       "Quantization format"): int8 codes with one symmetric fp32 scale per
 *       output row; W[o,k] = q[o,k] * scale[o], scale[o] = max|W[o,:]|/127.
 *         Wq    int8  [N, K], row-major
 *         scale float [N]
 *
 *   e4m3 ("RT-J -- FP8 E4M3 checkpoints", section "FP8 Format"): each weight
 *       matrix holds float8_e4m3fn values as they are, no scale: sign, 4 exponent
 *       bits (bias 7), 3 mantissa bits, subnormals m * 2^-9, largest 448; the
 *       codes S.1111.111 are NaN in the format and are not weights (the GEMM
 *       kernels read them as +-480).
 *         W     uint8 [N, K], row-major
 *
 * Activations X are fp32 [M, K] row-major and results Y are fp32 [M, N]
 * row-major.  There is no bias term (the cards keep biases in fp32 outside
 * the quantized projections).
 *
 * Conventions for every GEMM entry point:
 *   - Ownership: the caller allocates and owns every buffer it passes.  The
 *     library's only allocation is the activation workspace described at
 *     rt_workspace_bytes(); it never frees caller memory.
 *   - Pointers: X, Wq, scale(_min) and Y are DEVICE pointers on the current
 *     device; `stream` is a cudaStream_t (NULL = legacy default stream).
 *   - Execution: stream-ordered and asynchronous.  RT_OK means "validated and
 *     enqueued".  Conditions found later on the device (a bounded wait that
 *     gave up, an activation outside the fp16 range) are latched in a device
 *     status word read by rt_device_status().
 *   - Alignment: X, Y and Wq 16-byte aligned; scale_min 4-byte aligned (16
 *     for the TMA-fed kernels above 128 rows, see rt_qgemm_plan); scale
 *     4-byte aligned.  Otherwise RT_ERR_ALIGNMENT.
 *   - Shapes: M >= 0 (M == 0 is a no-op), N >= 1, K >= 1; q4 needs K % 32 == 0
 *     (the group size); q8 needs K % 16 == 0.  The tensor-core path also needs
 *     K % 64 == 0; RT_PATH_AUTO falls back to the SIMT path otherwise and an
 *     explicit RT_PATH_TC returns RT_ERR_UNSUPPORTED_SHAPE.
 *   - Aliasing: Y must not overlap X, Wq or the scales (RT_ERR_INVALID_ARG).
 *   - No C++ exception crosses this boundary.
 *   - Precision: the SIMT path dequantizes to fp32 and accumulates in fp32
 *     (max|Y - Y_exact| / max|Y_exact| <= 1e-5).  The tensor-core path rounds
 *     X and the exact dequantized q4 weights once to fp16 -- q8 codes are
 *     exact, their row scale is applied in fp32 after the MMA -- and
 *     accumulates in fp32 in TMEM (<= 4e-3; about 3e-4 on N(0,1) activations).
 *     fp16 operands hold |x| < 65520: an activation that rounds to infinity
 *     or is not finite makes the affected outputs infinite or NaN and latches
 *     RT_ERR_OPERAND_RANGE for rt_device_status(); such activations need the
 *     SIMT path.
 */
#ifndef RTQ_H
#define RTQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rt_status {
    RT_OK = 0,
    RT_ERR_INVALID_ARG = 1,       /* null pointer, negative size, overlap, bad n_grid */
    RT_ERR_ALIGNMENT = 2,         /* a pointer misses the alignment stated above */
    RT_ERR_UNSUPPORTED_SHAPE = 3, /* K not a multiple of the format's granule */
    RT_ERR_CUDA = 4,              /* a CUDA runtime call failed (launch, no device) */
    RT_ERR_DEVICE_TIMEOUT = 5,    /* a kernel's bounded wait expired (see rt_device_status) */
    RT_ERR_VALUE_RANGE = 6,       /* quantizer input not finite / outside binary16 range */
    RT_ERR_WORKSPACE = 7,         /* the workspace would have to grow inside a stream capture */
    RT_ERR_SCRATCH_LIMIT = 8,     /* rt_qgemm_noalloc: M * K * 2 > RT_NOALLOC_SCRATCH_BYTES */
    RT_ERR_OPERAND_RANGE = 9,     /* an activation was not a finite fp16 value (rt_device_status) */
    RT_ERR_UNSUPPORTED_DEVICE = 10, /* current device index >= 64, the library's per-device limit */
    RT_ERR_IO = 11,               /* a checkpoint file cannot be opened or mapped */
    RT_ERR_FORMAT = 12,           /* a checkpoint file or tensor is malformed */
    RT_ERR_NOT_FOUND = 13         /* a checkpoint has no tensor (or companion) of that name */
} rt_status;

/* Weight formats, where an entry point takes a `fmt` argument. */
typedef enum rt_format {
    RT_FMT_E4M3 = 3,    /* FP8 E4M3 codes [N, K], no scales (scales pointer unused, may be NULL) */
    RT_FMT_Q4 = 4,      /* q4 g32 codes [N, K/2] + binary16 (scale, min) [N, K/32, 2] */
    RT_FMT_Q8 = 8       /* q8 codes [N, K] + fp32 row scales [N] */
} rt_format;

typedef enum rt_path {
    RT_PATH_AUTO = 0,   /* SIMT for K % 64 != 0 or M <= 16 (q4) / M <= 1 (q8,
                           e4m3), else TC: the measured single-call crossover */
    RT_PATH_SIMT = 1,   /* fp32 CUDA-core kernels */
    RT_PATH_TC = 2      /* tcgen05 tensor-core kernels, fp16 operands, fp32 accumulate in TMEM */
} rt_path;            /* any other value: RT_ERR_INVALID_ARG */

/* Human-readable name of a status code; never NULL. */
const char *rt_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int rt_version(void);

/*
 * Y = X * dequant_q4(Wq, scale_min)^T.   (int4 card, "Quantization format")
 * X [M,K] fp32, Wq [N,K/2] u8, scale_min [N,K/32,2] binary16, Y [M,N] fp32.
 */
rt_status rt_qgemm_q4(const float *X, const uint8_t *Wq, const uint16_t *scale_min, float *Y,
                      int64_t M, int64_t N, int64_t K, int path, void *stream);

/*
 * Y = X * dequant_q8(Wq, scale)^T.   (int8 card, "Quantization format")
 * X [M,K] fp32, Wq [N,K] i8, scale [N] fp32, Y [M,N] fp32.
 */
rt_status rt_qgemm_q8(const float *X, const int8_t *Wq, const float *scale, float *Y,
                      int64_t M, int64_t N, int64_t K, int path, void *stream);

/*
 * Y = X * dequant(Wq, scales)^T + bias, any weight format, with an optional
 * fp32 bias fused into the epilogue (the cards keep biases in fp32 next to
 * the quantized weights: int4 card, "Quantization format").
 *   fmt     rt_format (scales unused for RT_FMT_E4M3 and may be NULL);
 *   bias    NULL, or fp32 [N] device memory, 4-byte aligned, not overlapping
 *           Y (RT_ERR_ALIGNMENT / RT_ERR_INVALID_ARG);
 * each output is fma(sum, row scale, bias[o]) rounded once (row scale 1
 * for q4 and e4m3).  Everything else as for rt_qgemm_q4 / rt_qgemm_q8 /
 * rt_gemm_e4m3, which are this call with bias NULL.
 */
rt_status rt_qgemm(int fmt, const float *X, const void *Wq, const void *scales, const float *bias,
                   float *Y, int64_t M, int64_t N, int64_t K, int path, void *stream);

/*
 * Y = X * W^T with W the FP8 E4M3 weights, converted exactly to the operand
 * type inside the GEMM.   (FP8 card, "FP8 Format")
 * X [M,K] fp32, W [N,K] uint8 float8_e4m3fn codes, Y [M,N] fp32.  K % 16 == 0;
 * everything else as for rt_qgemm_q8 (paths, kernels, precision: the SIMT
 * path is exact up to fp32 accumulation, the tensor-core path rounds X to
 * fp16 and keeps the weights exact).
 */
rt_status rt_gemm_e4m3(const float *X, const uint8_t *W, float *Y, int64_t M, int64_t N,
                       int64_t K, int path, void *stream);

/* Which path RT_PATH_AUTO takes for a GEMM of format fmt (rt_format) and
 * this shape: RT_PATH_SIMT or RT_PATH_TC; -1 for an unsupported shape. */
int rt_qgemm_auto_path(int fmt, int64_t M, int64_t N, int64_t K);

/* Kernels behind the paths:
 *   RT_KERNEL_SIMT            fp32 CUDA-core kernel, one thread per output row;
 *   RT_KERNEL_TC_W_STATIONARY tcgen05, one 128-row weight tile x up to 128
 *                             activation rows per CTA, converter warps load and
 *                             convert both operands (M <= 128, or shapes the
 *                             TMA kernels do not take); with one activation
 *                             tile, K is split over a cluster of up to 8 CTAs
 *                             whose partial sums are reduced in distributed
 *                             shared memory (deterministic order);
 *   RT_KERNEL_TC_X_RESIDENT   tcgen05, persistent CTAs keep a 192-row block of
 *                             activations in shared memory and stream TMA-staged
 *                             weight tiles past it (M > 128, K a multiple of
 *                             128 up to 512);
 *   RT_KERNEL_TC_W_STREAMED   tcgen05, persistent 128 x 192 tiles with both
 *                             operands TMA-staged (M > 128, other K);
 *   RT_KERNEL_TC_LIST         tcgen05, rt_qgemm_batch only: persistent CTAs
 *                             stream the weights of a whole list of
 *                             projections with the same M <= 128;
 *   RT_KERNEL_TC_X_RESIDENT_PAIR  the activation-resident product on pairs of
 *                             CTAs (one tcgen05 MMA over two SMs, 256 weight
 *                             rows x 192 activation rows), rounding X to fp16
 *                             inside the kernel (M >= 16384, K a multiple of
 *                             128 up to 512).
 * RT_KERNEL_TC_X_RESIDENT and RT_KERNEL_TC_W_STREAMED run an activation
 * pre-pass (X rounded once to fp16) into a per-(device, stream) workspace of
 * M * K * 2 bytes; RT_KERNEL_TC_X_RESIDENT_PAIR needs none. */
typedef enum rt_kernel {
    RT_KERNEL_SIMT = 1,
    RT_KERNEL_TC_W_STATIONARY = 2,
    RT_KERNEL_TC_X_RESIDENT = 3,
    RT_KERNEL_TC_W_STREAMED = 4,
    RT_KERNEL_TC_LIST = 5,
    RT_KERNEL_TC_X_RESIDENT_PAIR = 6
} rt_kernel;

/* The kernel a GEMM of this format, shape and path runs; -1 if rejected.
 * The plan assumes a 16-byte aligned q4 scale_min: the TMA-fed kernels
 * (RT_KERNEL_TC_X_RESIDENT, _W_STREAMED, _X_RESIDENT_PAIR) read it through a
 * tensor map, so a q4 call whose scale_min is only 4-byte aligned runs on
 * RT_KERNEL_TC_W_STATIONARY instead (same results, any M). */
int rt_qgemm_plan(int fmt, int64_t M, int64_t N, int64_t K, int path);

/*
 * Workspace.  RT_KERNEL_TC_X_RESIDENT and RT_KERNEL_TC_W_STREAMED stage the
 * activations, rounded to fp16, in a device buffer the library keeps per
 * (device, stream): rt_workspace_bytes() gives the size a GEMM needs
 * (M * K * 2 for those two kernels, 0 for the others, -1 for a rejected
 * shape).  The buffer grows on first need with
 * cudaMalloc; growth synchronizes that stream.  It cannot grow while the
 * stream is being captured into a CUDA graph -- such a call returns
 * RT_ERR_WORKSPACE -- so reserve the largest size first with
 * rt_workspace_reserve(bytes, stream).  rt_workspace_release() synchronizes
 * the current device and frees its workspaces.  Calls that share a stream
 * share its workspace in stream order.
 */
int64_t rt_workspace_bytes(int fmt, int64_t M, int64_t N, int64_t K, int path);
rt_status rt_workspace_reserve(int64_t bytes, void *stream);
rt_status rt_workspace_release(void);

/*
 * The same GEMM without any device allocation (the model cards have no
 * counterpart; this is a library convenience).  For callers that cannot
 * allocate device memory once they are running: a serving process whose own
 * pool already holds nearly all of HBM, so a late cudaMalloc would fail, or a
 * latency-bound loop that cannot take the stall of the workspace's growth
 * sync or of cudaFree.
 *
 * fmt = 4: Wq/scales are the q4 tensors of rt_qgemm_q4; fmt = 8: those of
 * rt_qgemm_q8.  X, Y, M, N, K, path and stream, validation and results are
 * as for rt_qgemm_q4/q8, and the same kernel runs (rt_qgemm_plan).  The
 * kernels that stage fp16 activations (RT_KERNEL_TC_X_RESIDENT,
 * RT_KERNEL_TC_W_STREAMED) use one file-scope device array of
 * RT_NOALLOC_SCRATCH_BYTES (16 MiB) per device instead of the per-stream
 * workspace; such a problem whose M * K * 2 exceeds it returns
 * RT_ERR_SCRATCH_LIMIT and launches nothing (for example M * K up to 8M
 * elements, M = 4096 x K = 2048).  The other kernels need no scratch.
 *
 * Set-up: the first call on a device that passes validation looks up
 * the array's device address, which may load the library's module; make
 * that first call before any stream capture.  No call allocates: no
 * cudaMalloc, cudaFree or allocating library routine.
 *
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents; each call writes all of the scratch it reads before
 * reading it.  Calls in one stream are ordered; calls that can overlap on
 * the GPU (different streams, or host threads without ordering) race on the
 * array and give wrong results.
 */
#define RT_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
rt_status rt_qgemm_noalloc(int fmt, const float *X, const void *Wq, const void *scales, float *Y,
                           int64_t M, int64_t N, int64_t K, int path, void *stream);

/*
 * A list of independent projections with the same M in one call.  The model
 * cards have no such call: it batches the projection they define (each entry
 * is exactly rt_qgemm_q4 or rt_qgemm_q8 on its own buffers) so that many
 * small-M projections -- the weight-bandwidth-bound regime, where a single
 * projection's weights stream in less time than a launch takes -- overlap
 * their weight streams instead of paying one launch and one dependency chain
 * each.
 *
 *   fmt       4: Wq/scales are q4 tensors as for rt_qgemm_q4;
 *             8: q8 tensors as for rt_qgemm_q8;
 *             3: Wq are e4m3 codes as for rt_gemm_e4m3 (scales unused).
 *   reserved  must be 0.
 *   bias      NULL, or an fp32 [N] bias added in the epilogue (rt_qgemm).
 *   X, Y      fp32 [M, K] / [M, N] device buffers of this projection.
 *
 * Validation: every entry as for rt_qgemm_q4/q8 (the same statuses); in
 * addition no entry's Y may overlap any other entry's X, Wq, scales, bias or Y
 * (RT_ERR_INVALID_ARG), since the entries may run concurrently; X, Wq and
 * scales may be shared between entries.  All entries are checked before
 * anything is enqueued.  count == 0 or M == 0 is a no-op.
 *
 * Route (rt_qgemm_batch_plan): with 1 <= M <= 128 on the tensor-core path
 * (RT_PATH_AUTO above the SIMT range, or RT_PATH_TC), every entry's K a
 * multiple of 128 (q4) or 64 (q8 and e4m3) and every q4 scale_min 16-byte
 * aligned, the list runs as RT_KERNEL_TC_LIST: one pre-pass launch rounds
 * each distinct (X, K) once to fp16 into the stream's workspace, then
 * persistent launches of up to 64 entries each stream the entries' weights
 * through every SM.  Each 128-row tile of an entry is computed over all of K
 * by one CTA (K > 512 in 512-wide chunks into one accumulator), so results
 * are deterministic.  Workspace (rt_workspace_reserve applies): per distinct
 * (X, K) M16 * K * 2 bytes (256-byte aligned), with M16 = M rounded up to 16.
 * The host encodes a TMA tensor map per entry's weights (cached per thread
 * by pointer and shape); Wq must be 16-byte aligned.  Under
 * RT_PATH_AUTO this happens only when the entries hold at least as many
 * 128-row weight tiles as the GPU has SMs.  Otherwise the entries run as
 * rt_qgemm calls would, except that entries which take
 * RT_KERNEL_TC_X_RESIDENT (M > 128) share launches: in list order, up to
 * four of them at a time (q4 scale_min 16-byte aligned) run as one pre-pass
 * launch that rounds each one's X into its own slice of the stream's
 * workspace and one launch of the activation-resident kernel that walks all
 * their tiles, so they share one pipeline fill and drain and one wave tail.
 * A grouped entry gets the bits a single rt_qgemm call would give.  The other
 * entries that stage X (RT_KERNEL_TC_W_STREAMED, or an activation-resident
 * entry left alone) then have their pre-passes run on a second stream that the
 * library keeps per (device, stream), beside the first shared launch, and
 * their GEMMs follow the shared launches on `stream` (the two streams are
 * joined with events, so stream order and graph capture hold; the second
 * stream is created on the first such call outside a capture, and a call
 * inside a capture before that runs the pre-passes in order on `stream`).
 * Workspace of such a list: the sum of M * K * 2 over the largest launch's
 * entries plus M * K * 2 of every other entry that stages X (one slice
 * each); without the second stream, the larger of the two parts.  Results are those of the tensor-core path (<= 4e-3) and do
 * not depend on the entries' order.
 */
typedef struct rt_qproj {
    int32_t fmt;
    int32_t reserved;
    const float *X;
    const void *Wq;
    const void *scales;
    const float *bias;
    float *Y;
    int64_t N;
    int64_t K;
} rt_qproj;

rt_status rt_qgemm_batch(const rt_qproj *list, int count, int64_t M, int path, void *stream);

/* RT_KERNEL_TC_LIST if rt_qgemm_batch runs this list as list launches, 0 if
 * it makes one call per entry, -1 if it rejects the list.  Host-only. */
int rt_qgemm_batch_plan(const rt_qproj *list, int count, int64_t M, int path);

/*
 * One RT-J block's quantized projection set, following the mixed-precision
 * recipe of the int4 card ("Quantization format": wq/wk/wv/wg and ffn.w1/w3
 * in q4 g32, the residual-writing wo and ffn.w2 in q8 per-row):
 *   qkvg : q4, N = 4*d_model, K = d_model  (rows wq | wk | wv | wg)
 *   wo   : q8, N = d_model,   K = d_model
 *   w13  : q4, N = 2*d_ff,    K = d_model  (rows w1 | w3)
 *   w2   : q8, N = d_model,   K = d_ff
 * All pointers are device pointers.  The four products are independent (each
 * reads its own input; two inputs may be the same buffer).  Y_qkvg
 * [M, 4*d_model], Y_o [M, d_model], Y_13 [M, 2*d_ff], Y_2 [M, d_model].
 *
 * Launches: where all four products take RT_KERNEL_TC_W_STATIONARY with one
 * activation tile (1 <= M <= 128 on the tensor-core path: RT_PATH_AUTO above
 * the SIMT range, or RT_PATH_TC), one grouped launch of that
 * kernel computes all four: each CTA takes a 128-row weight tile of one of
 * the projections and a slice of its K; each projection splits K by its own
 * factor (so w2, with four times the K of the others, splits four times as
 * far) and reduces the slices in distributed shared memory in a fixed order.
 * Otherwise they run on `stream` as rt_qgemm_batch runs the list (qkvg, wo,
 * w13, w2) on its per-entry route: the projections that take
 * RT_KERNEL_TC_X_RESIDENT (128 < M < 16384, K <= 512: qkvg, wo and w13 of
 * RT-J) share one pre-pass launch and one activation-resident launch, the
 * others run one call each, as rt_qgemm_q4/q8 would, their pre-passes on the
 * second stream beside the shared launch (see rt_qgemm_batch).  Workspace:
 * the sum of M * K * 2 over the projections that share the launch plus
 * M * K * 2 of each other call that stages X (M = 4096 RT-J: 29.4 MB).
 *
 * Validation: each product as in rt_qgemm_q4/q8; in addition no output may
 * overlap another projection's output, activations, codes or scales
 * (RT_ERR_INVALID_ARG), since the products may run concurrently.  All four
 * are checked before anything is enqueued, so an error status means nothing
 * was launched.
 */
typedef struct rt_qblock {
    const uint8_t *qkvg;   const uint16_t *qkvg_sm;
    const int8_t *wo;      const float *wo_s;
    const uint8_t *w13;    const uint16_t *w13_sm;
    const int8_t *w2;      const float *w2_s;
    int64_t d_model;
    int64_t d_ff;
} rt_qblock;

rt_status rt_qblock_project(const rt_qblock *blk, int64_t M,
                            const float *X_qkvg, const float *X_o, const float *X_ffn,
                            const float *X_w2, float *Y_qkvg, float *Y_o, float *Y_13,
                            float *Y_2, int path, void *stream);

/* 1 if rt_qblock_project runs a block of these sizes as one grouped launch,
 * 0 if it makes one call per projection, -1 if it rejects the sizes or path.
 * Host-only; touches no device. */
int rt_qblock_fused(int64_t M, int64_t d_model, int64_t d_ff, int path);

/* How rt_qblock_project (rt_qblock_route) or rt_qblock_project_fmt
 * (rt_qblock_route_fmt) runs this block at M rows on `path`: the sum of
 *   RT_ROUTE_GROUPED_SMALL_M   one grouped launch of the weight-stationary
 *                              kernel (1 <= M <= 128 on the tensor-core path);
 *   RT_ROUTE_X_RESIDENT_GROUP  the projections that take
 *                              RT_KERNEL_TC_X_RESIDENT share one pre-pass
 *                              launch and one launch of that kernel;
 *   RT_ROUTE_SIDE_PREPASS      the other projections' pre-passes run on a
 *                              second stream beside that launch (when the
 *                              pre-pass's blocks fit on the SMs beside its
 *                              CTAs), and their GEMMs start without waiting
 *                              for it;
 * 0 if the projections run one call after another; -1 if the block, M or
 * path is rejected.  Reads the weights' scale pointers (alignment) and no
 * device memory; RT_ROUTE_SIDE_PREPASS asks the CUDA runtime for the
 * kernels' register counts, so it is never set without a device. */
typedef enum rt_route {
    RT_ROUTE_GROUPED_SMALL_M = 1,
    RT_ROUTE_X_RESIDENT_GROUP = 2,
    RT_ROUTE_SIDE_PREPASS = 4
} rt_route;
int rt_qblock_route(const rt_qblock *blk, int64_t M, int path);

/*
 * The same block projection set with each projection's format chosen by the
 * caller, e.g. the int8 card's all-int8 (Q8_0-style) recipe ("RT-J -- int8
 * (Q8_0-style) quantized checkpoints", section "Quantization format": every
 * block projection wq/wk/wv/wg, wo, ffn.w1/w2/w3 stored as I8 with a
 * per-output-row fp32 scale), where qkvg is a q8 [4*d_model, d_model] tensor
 * and w13 a q8 [2*d_ff, d_model] tensor.
 *   fmt       4: Wq u8 [N, K/2] and scales binary16 [N, K/32, 2] (q4);
 *             8: Wq i8 [N, K] and scales fp32 [N] (q8);
 *             3: Wq u8 [N, K] float8_e4m3fn codes, scales unused (the FP8
 *                card's recipe: every block projection in e4m3);
 *   reserved  must be 0;
 *   bias      NULL, or the projection's fp32 [N] bias, added in the
 *             epilogue as in rt_qgemm.
 * Shapes, outputs, launches, validation and errors are those of
 * rt_qblock_project; rt_qblock_project is this call with the int4 card's
 * mixed recipe (qkvg and w13 q4, wo and w2 q8).
 */
typedef struct rt_qweight {
    int32_t fmt;
    int32_t reserved;
    const void *Wq;
    const void *scales;
    const float *bias;
} rt_qweight;

typedef struct rt_qblock_fmt {
    rt_qweight qkvg, wo, w13, w2;
    int64_t d_model;
    int64_t d_ff;
} rt_qblock_fmt;

rt_status rt_qblock_project_fmt(const rt_qblock_fmt *blk, int64_t M,
                                const float *X_qkvg, const float *X_o, const float *X_ffn,
                                const float *X_w2, float *Y_qkvg, float *Y_o, float *Y_13,
                                float *Y_2, int path, void *stream);

/* As rt_qblock_fused for a block with the formats of `blk` (host-only). */
int rt_qblock_fused_fmt(const rt_qblock_fmt *blk, int64_t M, int path);
int rt_qblock_route_fmt(const rt_qblock_fmt *blk, int64_t M, int path);

/*
 * Host-side quantizers (HOST pointers, caller-allocated outputs, synchronous,
 * deterministic, thread-safe; several threads may work inside one call).
 *
 * rt_quantize_q4_g32 (int4 card, "Quantization format": min-MSE clip search
 * over the shrink grid 1.0 -> 0.8): for each row and group of 32, try the
 * n_grid shrink factors s_j = 1 - 0.2*j/(n_grid-1) (n_grid = 0 selects 21),
 * take (scale, min) = binary16((s_j*hi - s_j*lo)/15), binary16(s_j*lo) with
 * lo/hi the group's min/max, codes = clamp(round-half-even((w - min)/scale),
 * 0, 15) (all zero when the scale rounds to 0), keep the j of least squared
 * reconstruction error (smallest j on ties), pack the codes.
 * W fp32 [N,K] -> Wq u8 [N,K/2], scale_min binary16 [N,K/32,2].
 * Errors: RT_ERR_INVALID_ARG (null, negative size, n_grid < 0),
 * RT_ERR_UNSUPPORTED_SHAPE (K % 32), RT_ERR_VALUE_RANGE (a weight is not
 * finite or |w| > 65504).
 */
rt_status rt_quantize_q4_g32(const float *W, int64_t N, int64_t K, int n_grid,
                             uint8_t *Wq, uint16_t *scale_min);

/*
 * rt_quantize_q8_row (int8 card, "Quantization format"): scale[o] =
 * max|W[o,:]| / 127 (one fp32 division), q = clamp(round-half-even(w /
 * scale), -127, 127); a zero row gets scale 0 and zero codes.
 * W fp32 [N,K] -> Wq i8 [N,K], scale fp32 [N].  Errors: RT_ERR_INVALID_ARG,
 * RT_ERR_VALUE_RANGE (a weight is not finite).
 */
rt_status rt_quantize_q8_row(const float *W, int64_t N, int64_t K, int8_t *Wq, float *scale);

/*
 * rt_quantize_e4m3 (FP8 card, "FP8 Format": weight matrices hold
 * float8_e4m3fn values, no scale): each of the n weights to the nearest E4M3 value, ties to
 * the even code, the same rounding as PyTorch's float8_e4m3fn cast.  W fp32
 * [n] -> codes uint8 [n].  Errors: RT_ERR_INVALID_ARG, RT_ERR_VALUE_RANGE (a
 * weight is NaN or |w| > 464, which would round past 448; out is then
 * incomplete).
 */
rt_status rt_quantize_e4m3(const float *W, int64_t n, uint8_t *out);

/*
 * Dequantization exports (device pointers, stream-ordered).  They run the
 * same __device__ dequantization routines the GEMM kernels use, so tests can
 * check them bit for bit:
 *   *_f32  : W[o,k] rounded once to fp32 (the SIMT path's operand);
 *   q4_f16 : the exact value rounded once to fp16, stored as uint16 bits (the
 *            tensor-core path's q4 operand).
 * W_out is [N,K].  Same alignment and shape rules as the GEMMs.
 */
rt_status rt_dequant_q4_f32(const uint8_t *Wq, const uint16_t *scale_min, float *W_out,
                            int64_t N, int64_t K, void *stream);
rt_status rt_dequant_q8_f32(const int8_t *Wq, const float *scale, float *W_out,
                            int64_t N, int64_t K, void *stream);
rt_status rt_dequant_q4_f16(const uint8_t *Wq, const uint16_t *scale_min, uint16_t *W_out,
                            int64_t N, int64_t K, void *stream);
/* e4m3 codes -> their exact values in fp32 / in fp16 bits (the tensor-core
 * operand); K % 16 == 0, Wq and W_out 16-byte aligned. */
rt_status rt_dequant_e4m3_f32(const uint8_t *Wq, float *W_out, int64_t N, int64_t K,
                              void *stream);
rt_status rt_dequant_e4m3_f16(const uint8_t *Wq, uint16_t *W_out, int64_t N, int64_t K,
                              void *stream);

/*
 * Synchronizes `stream`, then reads and clears the current device's status
 * word, which the tensor-core kernels latch when one of their bounded waits
 * gives up (RT_ERR_DEVICE_TIMEOUT; outputs of that launch are undefined) or
 * when an activation is not a finite fp16 value after rounding
 * (RT_ERR_OPERAND_RANGE).  *device_status receives RT_OK or one of those two
 * (the timeout when both were latched).  Returns RT_ERR_CUDA if the
 * synchronization itself fails.
 */
rt_status rt_device_status(void *stream, int *device_status);

/*
 * Test hook for the device-side failure path (not for production use; the
 * model cards have no counterpart).  Synchronizes the current device, then
 * sets how its tensor-core kernels launched from now on behave:
 *   mode 0: normal operation;
 *   mode 1: in every CTA the first producer arrival is left out (a converter
 *           thread skips its arrival on the first stage, or the weight TMA
 *           thread never requests its first box), so a consumer's bounded
 *           wait runs out, the kernel winds down and latches
 *           RT_ERR_DEVICE_TIMEOUT.
 * wait_ns: bound of every mbarrier wait in nanoseconds; 0 restores the
 * default of 2 s.  RT_ERR_INVALID_ARG for another mode or a negative bound.
 * Restore rt_debug_inject(0, 0) before normal use.
 */
rt_status rt_debug_inject(int mode, int64_t wait_ns);

/*
 * Quantized checkpoints.  Both quantized cards ship their checkpoints as
 * ordinary safetensors files, which the engine's loader reads without
 * conversion, telling the format from the tensors' dtypes; the FP8 card
 * stores float8_e4m3fn weights the same way.  These calls read such a file
 * on the host (the model cards have no other interface to match):
 *
 *   rt_st_open          maps the file read-only and parses its header;
 *                       RT_ERR_IO if it cannot be opened or mapped,
 *                       RT_ERR_FORMAT if the header, a dtype, a shape or an
 *                       offset is malformed.  *out is NULL on error.
 *   rt_st_count         number of tensors in the file (-1 for NULL).
 *   rt_st_weight_find   the projection weight `name`, its format detected:
 *                         U8 [N, K/2] + "<name>.q4_scale" F16 [N, K/32, 2]
 *                           (or [N, K/16])                      -> RT_FMT_Q4
 *                         I8 [N, K] + "<name>.q_scale" F32 [N] (or [N, 1])
 *                                                               -> RT_FMT_Q8
 *                         F8_E4M3 [N, K]                        -> RT_FMT_E4M3
 *                       Pointers are HOST pointers into the mapping, valid
 *                       until rt_st_close, with no alignment guarantee (copy
 *                       them to device memory for the GEMMs); scales is NULL
 *                       for e4m3.  RT_ERR_NOT_FOUND if `name` or its
 *                       companion is missing, RT_ERR_FORMAT for another dtype
 *                       or inconsistent shapes, RT_ERR_UNSUPPORTED_SHAPE if the
 *                       weight is not a non-empty 2-D tensor.
 *   rt_st_close         unmaps the file (NULL is a no-op).
 * Files are only read; calls on distinct files may run concurrently.
 */
typedef struct rt_st_file rt_st_file;

typedef struct rt_st_weight {
    int32_t fmt;            /* rt_format */
    int32_t reserved;
    int64_t N, K;
    const void *codes;      /* code_bytes bytes */
    const void *scales;     /* scale_bytes bytes; NULL for e4m3 */
    int64_t code_bytes, scale_bytes;
} rt_st_weight;

rt_status rt_st_open(const char *path, rt_st_file **out);
int64_t rt_st_count(const rt_st_file *f);
rt_status rt_st_weight_find(const rt_st_file *f, const char *name, rt_st_weight *out);
void rt_st_close(rt_st_file *f);

#ifdef __cplusplus
}
#endif

#endif /* RTQ_H */
