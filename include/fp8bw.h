/*
 * fp8bw.h -- C ABI of the blockwise-FP8 training-linear library for B200
 * (sm_100a).
 *
 * What the library computes (Puro-2B report summaries):
 *   - arxiv-wiki summary of "Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX
 *     5090 within $5090", section "Approach", item (4): the Transformer's main
 *     linear operations run in blockwise FP8 E4M3, activations with one scale
 *     per 1-D group of 128 elements, weights with one scale per 128x128 block.
 *   - paperlayer.ai summary of the same report, Appendix C, "FP8
 *     implementation pipeline": the E4M3 GEMMs of the linear layers are forward
 *     propagation, data-gradient and weight-gradient; hidden/residual flow stays
 *     bf16.
 * The pages print no formula. The readings taken here:
 *   - group scale: amax = max |x| over the group; qscale = 448/amax and stored
 *     (dequantisation) scale s = amax/448, both fp32 round-to-nearest-even;
 *     amax == 0, or a qscale that overflows fp32, gives qscale = s = 1.
 *   - code = E4M3(x * qscale): one fp32 multiply, then round-to-nearest-even
 *     with saturation to +-448 (0x7E/0xFE).
 *   - GEMMs accumulate in fp32; every 128-long chunk of the contraction
 *     dimension is computed separately on the tensor cores and added into the
 *     fp32 accumulator times the product of its two scales; bf16 output (RNE).
 *
 * Conventions for every call:
 *   - All data pointers are DEVICE pointers owned by the caller. The library
 *     never allocates, frees or keeps them. Outputs must not alias inputs. A
 *     pointer may be NULL only when its buffer holds no element.
 *   - A call runs on the calling thread's current CUDA device: its pointers
 *     and `stream` must belong to that device (the library cannot tell which
 *     device a pointer belongs to; memory of another GPU is not supported).
 *   - bf16 tensors are passed as uint16_t bit patterns. FP8 codes are uint8_t
 *     OCP E4M3 codes. Scales are fp32.
 *   - Matrices are dense row-major (leading dimension = row length).
 *   - Every call is asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *     default stream) and returns an fp8bw_status. Argument errors are found
 *     on the host before anything is launched, and then nothing is written.
 *   - Limits: every dimension <= 2^30; a quantiser takes at most 65535 row
 *     tiles of 128 and fewer than 2^31 tiles of 128 x 128; a GEMM at most 2^30
 *     output tiles of 256 x 256 (else FP8BW_ERR_SHAPE).
 *   - Shapes: every dimension >= 0 and a multiple of 16. Dimensions that are
 *     not multiples of 128 give a short last group (its amax runs over the
 *     elements present) and a short last chunk. A zero dimension is a no-op,
 *     except a GEMM with an empty contraction, which writes zeros.
 *   - Pointers must be 16-byte aligned.
 *   - Scale layouts ("group-major, contiguous along the other dimension", so a
 *     128-row GEMM tile reads its 128 scales of one chunk in one 512-B run):
 *       row-wise 1x128 groups of X[rows, cols]  : s[ceil(cols/128)][rows]
 *       col-wise 128x1 groups of X[rows, cols]  : s_t[ceil(rows/128)][cols]
 *       128x128 blocks of W[n, k]               : s[ceil(n/128)][ceil(k/128)]
 *   - The kernels run only on compute capability 10.0 (B200, sm_100a); other
 *     devices get FP8BW_ERR_DEVICE.
 *   - Device-side waits are bounded: a wait that does not finish within about
 *     two seconds makes the kernel record FP8BW_ERR_DEVICE_TIMEOUT in a device
 *     flag and return; fp8bw_check_device_error() reads and clears that flag.
 */
#ifndef FP8BW_H
#define FP8BW_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp8bw_status {
    FP8BW_OK = 0,
    FP8BW_ERR_NULL = -1,           /* a required pointer is NULL */
    FP8BW_ERR_SHAPE = -2,          /* a dimension < 0 or not a multiple of 16 */
    FP8BW_ERR_ALIGN = -3,          /* a pointer is not 16-byte aligned */
    FP8BW_ERR_DEVICE = -4,         /* current device is not sm_100 */
    FP8BW_ERR_LAUNCH = -5,         /* the CUDA launch failed */
    FP8BW_ERR_DEVICE_TIMEOUT = -6, /* a bounded device-side wait expired */
    FP8BW_ERR_CUDA = -7,           /* another CUDA runtime/driver call failed */
    FP8BW_ERR_ALIAS = -8,          /* an output overlaps an input */
    FP8BW_ERR_SCALE = -9           /* a *_pow2 GEMM read a scale that is not
                                      a power of two (reported by
                                      fp8bw_check_device_error) */
} fp8bw_status;

/* Row-wise 1x128 quantisation of an activation or gradient X[rows, cols]
 * (groups along cols, the contraction dimension of fprop for X and of dgrad
 * for dY).
 *   x : bf16 [rows, cols]                         (in)
 *   q : E4M3 codes [rows, cols]                   (out)
 *   s : fp32 scales [ceil(cols/128)][rows]        (out)
 * Source: arxiv-wiki summary, Approach item (4) (activation 1-D groups of 128).
 * HBM traffic: 2 B read + 1 B + 4/128 B written per element. */
int fp8bw_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                           uint8_t* q, float* s, void* stream);

/* Column-wise 128x1 quantisation of X[rows, cols] (groups along rows, the
 * token dimension, which the weight-gradient GEMM contracts), with the codes
 * written transposed. If q_row and s_row are both non-NULL the same pass also
 * writes the row-wise 1x128 result (one read of X for both).
 *   x     : bf16 [rows, cols]                     (in)
 *   q_t   : E4M3 codes [cols, rows]               (out)
 *   s_t   : fp32 scales [ceil(rows/128)][cols]    (out)
 *   q_row : E4M3 codes [rows, cols] or NULL       (out)
 *   s_row : fp32 [ceil(cols/128)][rows] or NULL   (out)
 * Source: paperlayer.ai summary, Appendix C, "FP8 implementation pipeline"
 * (weight-gradient GEMM) with the 1-D group of 128 of the arxiv-wiki summary,
 * Approach item (4). Either both of q_row/s_row are NULL or neither. */
int fp8bw_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                           uint8_t* q_t, float* s_t, uint8_t* q_row,
                           float* s_row, void* stream);

/* 128x128 block quantisation of a weight W[n, k] (out x in).
 *   w   : bf16 [n, k]                             (in)
 *   q   : E4M3 codes [n, k]                       (out)
 *   s   : fp32 scales [ceil(n/128)][ceil(k/128)]  (out)
 *   q_t : E4M3 codes [k, n] (the same codes transposed, for dgrad) or NULL
 * Source: arxiv-wiki summary, Approach item (4) (weights in 128x128 blocks). */
int fp8bw_quantize_weight_block(const uint16_t* w, int64_t n, int64_t k,
                                uint8_t* q, float* s, uint8_t* q_t,
                                void* stream);

/* Several weights' 128x128 block quantisations in one launch (the weights of
 * a layer, quantised once per step): each job is exactly what
 * fp8bw_quantize_weight_block(w, n, k, q, s, q_t) computes; the tensors'
 * tiles are walked by one persistent grid, so small weights share one
 * launch's ramp and tail.
 *   jobs  : HOST array of `count` job descriptions (read during the call
 *           only); each job's pointers are device pointers as above.
 *   count : 0..8 (0 is a no-op; more is FP8BW_ERR_SHAPE).
 * Errors: a job's own checks as fp8bw_quantize_weight_block; besides, no
 * output of any job may overlap any job's input or any other output
 * (FP8BW_ERR_ALIAS). Nothing is launched when a check fails. */
typedef struct fp8bw_weight_block_job {
    const uint16_t* w;   /* bf16 [n, k]                                    */
    int64_t n, k;
    uint8_t* q;          /* E4M3 codes [n, k]                              */
    float* s;            /* fp32 scales [ceil(n/128)][ceil(k/128)]         */
    uint8_t* q_t;        /* E4M3 codes [k, n] (transposed) or NULL         */
} fp8bw_weight_block_job;

int fp8bw_quantize_weight_block_batch(const fp8bw_weight_block_job* jobs,
                                      int count, void* stream);

/* fprop: Y[m, n] = bf16( sum_c sX[c][m] * sW[n/128][c] *
 *                        sum_{kk in chunk c} qX[m, kk] * qW[n, kk] )
 *   qx, sx : row-wise quantised X: [m, k], [ceil(k/128)][m]
 *   qw, sw : block-quantised W: [n, k], [ceil(n/128)][ceil(k/128)]
 *   y      : bf16 [m, n]                          (out)
 * Source: paperlayer.ai summary, Appendix C ("forward propagation"). */
int fp8bw_gemm_fprop(const uint8_t* qx, const float* sx, const uint8_t* qw,
                     const float* sw, int64_t m, int64_t n, int64_t k,
                     uint16_t* y, void* stream);

/* dgrad: dX[m, k] = bf16( sum_c sdY[c][m] * sW[c][k/128] *
 *                         sum_{nn in chunk c} qdY[m, nn] * qW[nn, k] )
 *   qdy, sdy : row-wise quantised dY: [m, n], [ceil(n/128)][m]
 *   qw       : the weight codes, either transposed qW^T [k, n]
 *              (qw_is_transposed = 1, as written by fp8bw_quantize_weight_block
 *              into q_t) or as stored, qW [n, k] (qw_is_transposed = 0)
 *   sw       : block scales [ceil(n/128)][ceil(k/128)] (the same blocks as
 *              fprop: a square block is transpose invariant)
 *   dx       : bf16 [m, k]                        (out)
 * Source: paperlayer.ai summary, Appendix C ("data-gradient"). */
int fp8bw_gemm_dgrad(const uint8_t* qdy, const float* sdy, const uint8_t* qw,
                     int qw_is_transposed, const float* sw, int64_t m,
                     int64_t n, int64_t k, uint16_t* dx, void* stream);

/* wgrad: dW[n, k] = bf16( sum_c sdYt[c][n] * sXt[c][k] *
 *                         sum_{mm in chunk c} qdYt[n, mm] * qXt[k, mm] )
 *   qdy_t, sdy_t : col-wise quantised dY: [n, m], [ceil(m/128)][n]
 *   qx_t,  sx_t  : col-wise quantised X:  [k, m], [ceil(m/128)][k]
 *   dw           : bf16 [n, k]                    (out)
 * Source: paperlayer.ai summary, Appendix C ("weight-gradient"). */
int fp8bw_gemm_wgrad(const uint8_t* qdy_t, const float* sdy_t,
                     const uint8_t* qx_t, const float* sx_t, int64_t m,
                     int64_t n, int64_t k, uint16_t* dw, void* stream);

/* wgrad with an fp32 weight gradient: the same sum as fp8bw_gemm_wgrad, kept
 * in fp32 (no bf16 rounding), for the fp32 main-grad of mixed-precision
 * training.
 *   accumulate == 0 : dW := P           (dw is write-only)
 *   accumulate != 0 : dW := fp32(dW + P) element-wise, P being the fp32 sum
 *                     above; dw must hold the previous gradient (e.g. the
 *                     other micro-batches' sum). The add is done in memory,
 *                     by the TMA unit, once per element per call.
 *   dw : fp32 [n, k], caller-owned device memory, 16-byte aligned, must not
 *        overlap any input. Other arguments and errors as fp8bw_gemm_wgrad;
 *        m == 0 writes zeros (accumulate == 0) or leaves dw unchanged.
 * Source: paperlayer.ai summary, Appendix C, "FP8 implementation pipeline"
 * (gradients are kept in FP32; the weight-gradient GEMM is one of the FP8
 * GEMMs). */
int fp8bw_gemm_wgrad_f32(const uint8_t* qdy_t, const float* sdy_t,
                         const uint8_t* qx_t, const float* sx_t, int64_t m,
                         int64_t n, int64_t k, float* dw, int accumulate,
                         void* stream);

/* Several weight gradients in one launch (the linears of a layer, whose
 * backward passes all contract over the same tokens): each job is exactly
 * what fp8bw_gemm_wgrad (bf16 dW) or fp8bw_gemm_wgrad_f32 (fp32 dW, stored
 * or, with accumulate != 0, added into dw) computes for its arguments; the
 * jobs' output tiles share one persistent grid, so the last wave of one
 * problem is filled with tiles of the next.
 *   jobs       : HOST array of `count` job descriptions (read during the call
 *                only); pointers are device pointers with the layouts of
 *                fp8bw_gemm_wgrad; dw is bf16 [n, k] for
 *                fp8bw_gemm_wgrad_batch, fp32 [n, k] for the _f32 form.
 *   count      : 0..4 (0 is a no-op; more is FP8BW_ERR_SHAPE).
 *   accumulate : the same for every job.
 * Errors: a job's own checks as the single-problem call; all jobs must have
 * the same m (FP8BW_ERR_SHAPE); no dw may overlap any job's input or another
 * dw (FP8BW_ERR_ALIAS). Nothing is launched when a check fails.
 * Source: paperlayer.ai summary, Appendix C, "FP8 implementation pipeline"
 * (the weight-gradient GEMM of each linear). */
typedef struct fp8bw_wgrad_job {
    const uint8_t* qdy_t;   /* col-wise quantised dY: codes [n, m]           */
    const float* sdy_t;     /*   scales [ceil(m/128)][n]                     */
    const uint8_t* qx_t;    /* col-wise quantised X: codes [k, m]            */
    const float* sx_t;      /*   scales [ceil(m/128)][k]                     */
    int64_t m, n, k;
    void* dw;               /* bf16 or fp32 [n, k], per the entry point      */
} fp8bw_wgrad_job;

int fp8bw_gemm_wgrad_batch(const fp8bw_wgrad_job* jobs, int count,
                           void* stream);
int fp8bw_gemm_wgrad_f32_batch(const fp8bw_wgrad_job* jobs, int count,
                               int accumulate, void* stream);

/* fprop / dgrad that also quantise their own bf16 output row-wise, for a
 * linear that consumes it next: the same y (dx) as fp8bw_gemm_fprop
 * (fp8bw_gemm_dgrad), plus exactly what fp8bw_quantize_rowwise would write
 * for that bf16 output, without reading it back from memory.
 *   qy, sy   : E4M3 codes [m, n] and scales [ceil(n/128)][m] of y (out)
 *   qdx, sdx : E4M3 codes [m, k] and scales [ceil(k/128)][m] of dx (out)
 * Other arguments and errors as the calls without the suffix; the extra
 * outputs are required (non-NULL when non-empty), 16-byte aligned and must
 * not overlap any input or each other.
 * Source: paperlayer.ai summary, Appendix C, "FP8 implementation pipeline"
 * (bf16 hidden flow between E4M3 GEMMs; the 1x128 row groups of the
 * arxiv-wiki summary, Approach item (4)). */
int fp8bw_gemm_fprop_quant(const uint8_t* qx, const float* sx,
                           const uint8_t* qw, const float* sw, int64_t m,
                           int64_t n, int64_t k, uint16_t* y, uint8_t* qy,
                           float* sy, void* stream);
int fp8bw_gemm_dgrad_quant(const uint8_t* qdy, const float* sdy,
                           const uint8_t* qw, int qw_is_transposed,
                           const float* sw, int64_t m, int64_t n, int64_t k,
                           uint16_t* dx, uint8_t* qdx, float* sdx,
                           void* stream);

/* fprop / dgrad that quantise their own bf16 output both ways, as
 * fp8bw_quantize_colwise with q_row/s_row would: the row-wise codes and
 * scales of the calls above, plus the column-wise 128x1 codes written
 * transposed and their scales -- what the next linear's fprop (row-wise) and
 * wgrad (column-wise, token groups) consume, without reading the output back
 * from memory.
 *   qy_t, sy_t   : E4M3 codes [n, m] (transposed) and scales
 *                  [ceil(m/128)][n] of y (out)
 *   qdx_t, sdx_t : E4M3 codes [k, m] and scales [ceil(m/128)][k] of dx (out)
 * The column groups are the 128-row (token) blocks of the output; a short
 * last block is a short group (its amax runs over the rows present). Other
 * arguments and errors as fp8bw_gemm_fprop_quant / fp8bw_gemm_dgrad_quant;
 * all four extra outputs are required (non-NULL when non-empty), 16-byte
 * aligned and must not overlap any input or each other.
 * Source: paperlayer.ai summary, Appendix C, "FP8 implementation pipeline"
 * (bf16 flow between the E4M3 GEMMs; the weight-gradient GEMM contracts over
 * tokens) with the 1-D 128-groups of the arxiv-wiki summary, Approach
 * item (4). */
int fp8bw_gemm_fprop_quant_rowcol(const uint8_t* qx, const float* sx,
                                  const uint8_t* qw, const float* sw,
                                  int64_t m, int64_t n, int64_t k, uint16_t* y,
                                  uint8_t* qy, float* sy, uint8_t* qy_t,
                                  float* sy_t, void* stream);
int fp8bw_gemm_dgrad_quant_rowcol(const uint8_t* qdy, const float* sdy,
                                  const uint8_t* qw, int qw_is_transposed,
                                  const float* sw, int64_t m, int64_t n,
                                  int64_t k, uint16_t* dx, uint8_t* qdx,
                                  float* sdx, uint8_t* qdx_t, float* sdx_t,
                                  void* stream);

/* ------------------------------------------------------------------------
 * Power-of-two scales on the tensor cores' block scaling.
 *
 * The pages fix blockwise E4M3 with 1x128 activation groups and 128x128
 * weight blocks, each with one scale (arxiv-wiki summary, "Approach" item
 * (4)), and say the grouping and scaling follow the DeepSeek-V3 approach
 * (same page, developer notes, bullet 3); they do not fix the form of the
 * scale. These entry points use power-of-two scales: s = 2^E with E the
 * smallest integer such that 448 * 2^E >= amax (E >= -127; an all-zero group
 * gets s = 1), codes E4M3(x * 2^-E). With such scales the B200 tensor cores
 * apply the scales themselves (UE8M0 block scaling) and accumulate the whole
 * contraction in fp32, so the GEMMs need no per-chunk promotion.
 *
 * Arguments, layouts, ownership and errors are those of the entry points
 * without the suffix. Scales stay fp32 (exact powers of two) in the same
 * layouts; the *_pow2 GEMMs accept only such scales (anything else makes the
 * next fp8bw_check_device_error return FP8BW_ERR_SCALE, and that output is
 * undefined). The codes of a *_pow2 quantiser feed only *_pow2 GEMMs.
 * ------------------------------------------------------------------------ */
int fp8bw_quantize_rowwise_pow2(const uint16_t* x, int64_t rows, int64_t cols,
                                uint8_t* q, float* s, void* stream);
int fp8bw_quantize_colwise_pow2(const uint16_t* x, int64_t rows, int64_t cols,
                                uint8_t* q_t, float* s_t, uint8_t* q_row,
                                float* s_row, void* stream);
int fp8bw_quantize_weight_block_pow2(const uint16_t* w, int64_t n, int64_t k,
                                     uint8_t* q, float* s, uint8_t* q_t,
                                     void* stream);
int fp8bw_quantize_weight_block_batch_pow2(const fp8bw_weight_block_job* jobs,
                                           int count, void* stream);
int fp8bw_gemm_fprop_pow2(const uint8_t* qx, const float* sx,
                          const uint8_t* qw, const float* sw, int64_t m,
                          int64_t n, int64_t k, uint16_t* y, void* stream);
int fp8bw_gemm_dgrad_pow2(const uint8_t* qdy, const float* sdy,
                          const uint8_t* qw, int qw_is_transposed,
                          const float* sw, int64_t m, int64_t n, int64_t k,
                          uint16_t* dx, void* stream);
int fp8bw_gemm_wgrad_pow2(const uint8_t* qdy_t, const float* sdy_t,
                          const uint8_t* qx_t, const float* sx_t, int64_t m,
                          int64_t n, int64_t k, uint16_t* dw, void* stream);

/* Power-of-two wgrad with an fp32 weight gradient (the power-of-two form of
 * fp8bw_gemm_wgrad_f32): the fp32 sum that fp8bw_gemm_wgrad_pow2 rounds to
 * bf16, stored (accumulate == 0) or added
 * element-wise into dw (accumulate != 0: dW := fp32(dW + P), one add per
 * element by the TMA unit), as fp8bw_gemm_wgrad_f32 does for the other scale
 * form. dw: fp32 [n, k], caller-owned, 16-byte aligned, not overlapping any
 * input. Source: paperlayer.ai summary, Appendix C, "FP8 implementation
 * pipeline" (gradients kept in FP32). */
int fp8bw_gemm_wgrad_f32_pow2(const uint8_t* qdy_t, const float* sdy_t,
                              const uint8_t* qx_t, const float* sx_t,
                              int64_t m, int64_t n, int64_t k, float* dw,
                              int accumulate, void* stream);
/* The batched forms (one launch per job: the power-of-two kernel takes one
 * problem at a time); checks and errors as fp8bw_gemm_wgrad_batch. */
int fp8bw_gemm_wgrad_batch_pow2(const fp8bw_wgrad_job* jobs, int count,
                                void* stream);
int fp8bw_gemm_wgrad_f32_batch_pow2(const fp8bw_wgrad_job* jobs, int count,
                                    int accumulate, void* stream);

/* Synchronises `stream`, then returns FP8BW_ERR_DEVICE_TIMEOUT if any kernel
 * of this library on the current device recorded an expired wait since the
 * last call, FP8BW_ERR_SCALE if a *_pow2 GEMM recorded a scale that is not a
 * power of two (and clears the record), else FP8BW_OK (or FP8BW_ERR_CUDA if
 * the synchronisation itself failed). */
int fp8bw_check_device_error(void* stream);

/* Test of the error path of the library's bounded device-side waits: one
 * block waits on a barrier that nothing completes; after limit_ns (0 to 1e9
 * ns, else FP8BW_ERR_SHAPE) the wait gives up and records a timeout, so the
 * next fp8bw_check_device_error returns FP8BW_ERR_DEVICE_TIMEOUT (and clears
 * it). Nothing faults or hangs; the context stays usable. Writes nothing but
 * the error record. (No counterpart on the pages: robustness of this
 * library.) */
int fp8bw_selftest_wait_timeout(int64_t limit_ns, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* fp8bw_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int fp8bw_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FP8BW_H */
