/*
 * fp8bw_oracle.h -- plain CPU reference for the blockwise-FP8 training linear.
 *
 * TEST INFRASTRUCTURE. This header belongs to the oracle alone. Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg may call these
 * functions; the library's product path never does, and the oracle shares no
 * code, header, table or helper with the CUDA kernels.
 *
 * What is computed (sources: the Puro-2B report summaries):
 *   - "Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within $5090"
 *     (arxiv-wiki summary), section "Approach", item (4): the main linear
 *     operations run in blockwise FP8 E4M3; activations carry one scale per 1-D
 *     group of 128 elements, weights one scale per 128x128 block.
 *   - the same report on paperlayer.ai, Appendix C, "FP8 implementation
 *     pipeline": the linear-layer GEMMs in E4M3 are forward propagation,
 *     data-gradient and weight-gradient.
 * The pages do not print the scale formula, rounding, saturation or the
 * accumulation interval; the readings used here are:
 *   scale      : qscale = 448/amax (fp32, RNE), stored scale s = amax/448;
 *                amax == 0 or a non-finite qscale gives qscale = s = 1.
 *   encode     : t = x*qscale (one fp32 multiply), then E4M3 round-to-nearest-
 *                even with saturation to +-448 (0x7E / 0xFE).
 *   GEMM       : every 128-long chunk c of the contraction dimension yields an
 *                exact partial P_c of decoded codes, scaled by the two scales of
 *                that chunk and summed in fp64 over chunks.
 *
 * Conventions: bf16 data is passed as raw uint16 bit patterns; all matrices are
 * dense row-major; dimensions need not be multiples of 128 (a short last group
 * takes its amax over the elements present). Scale layouts:
 *   row-wise 1x128   : s[g][row]       (g = col/128, rows contiguous)
 *   col-wise 128x1   : s_t[g][col]     (g = row/128, cols contiguous)
 *   weight 128x128   : s[nb][kb]       (row-major over blocks)
 * Return value of the int functions: 0 on success, -1 on bad arguments.
 */
#ifndef FP8BW_ORACLE_H
#define FP8BW_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* E4M3 (OCP FP8, bias 7, no infinities, 0x7F/0xFF NaN). */
double  orc_e4m3_decode(uint8_t code);
uint8_t orc_e4m3_encode(float t);
void    orc_e4m3_encode_array(const float* t, int64_t count, uint8_t* out);

/* Group scale pair from an amax (see header comment). */
void orc_group_scale(float amax, float* qscale, float* s);
/* Power-of-two variant: s = 2^E, E the smallest integer with 448 * 2^E >=
 * amax, clamped to [-127, 127]; qscale = 2^-E; amax == 0 or non-finite gives
 * qscale = s = 1. */
void orc_group_scale_pow2(float amax, float* qscale, float* s);

/* bf16 helpers (raw bit patterns). */
float    orc_bf16_to_float(uint16_t b);
uint16_t orc_bf16_round(double v);

/* Quantisers. */
int orc_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                         uint8_t* q, float* s);
int orc_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                         uint8_t* q_t, float* s_t);
int orc_quantize_weight_block(const uint16_t* w, int64_t n, int64_t k,
                              uint8_t* q, float* s, uint8_t* q_t);
/* The same quantisers with power-of-two scales (orc_group_scale_pow2). */
int orc_quantize_rowwise_pow2(const uint16_t* x, int64_t rows, int64_t cols,
                              uint8_t* q, float* s);
int orc_quantize_colwise_pow2(const uint16_t* x, int64_t rows, int64_t cols,
                              uint8_t* q_t, float* s_t);
int orc_quantize_weight_block_pow2(const uint16_t* w, int64_t n, int64_t k,
                                   uint8_t* q, float* s, uint8_t* q_t);

/* GEMMs, full output.  acc and bound are fp64 [rows_out][cols_out]; bound is
 * sum_k |a_k * b_k| of the dequantised operands (may be NULL). nthreads <= 1
 * runs on the calling thread. */
int orc_gemm_fprop(const uint8_t* qx, const float* sx, const uint8_t* qw,
                   const float* sw, int64_t m, int64_t n, int64_t k,
                   double* acc, double* bound, int nthreads);
int orc_gemm_dgrad(const uint8_t* qdy, const float* sdy, const uint8_t* qw,
                   const float* sw, int64_t m, int64_t n, int64_t k,
                   double* acc, double* bound, int nthreads);
int orc_gemm_wgrad(const uint8_t* qdy_t, const float* sdy_t,
                   const uint8_t* qx_t, const float* sx_t, int64_t m,
                   int64_t n, int64_t k, double* acc, double* bound,
                   int nthreads);

/* GEMMs at a list of output points (i[p], j[p]), for sampled checks at sizes
 * where the full product is too slow on the CPU. */
int orc_gemm_fprop_points(const uint8_t* qx, const float* sx, const uint8_t* qw,
                          const float* sw, int64_t m, int64_t n, int64_t k,
                          const int64_t* pi, const int64_t* pj, int64_t npts,
                          double* acc, double* bound, int nthreads);
int orc_gemm_dgrad_points(const uint8_t* qdy, const float* sdy,
                          const uint8_t* qw, const float* sw, int64_t m,
                          int64_t n, int64_t k, const int64_t* pi,
                          const int64_t* pj, int64_t npts, double* acc,
                          double* bound, int nthreads);
int orc_gemm_wgrad_points(const uint8_t* qdy_t, const float* sdy_t,
                          const uint8_t* qx_t, const float* sx_t, int64_t m,
                          int64_t n, int64_t k, const int64_t* pi,
                          const int64_t* pj, int64_t npts, double* acc,
                          double* bound, int nthreads);

#ifdef __cplusplus
}
#endif
#endif
