// quant.cuh -- E4M3 quantisers for sm_100a (HBM-bound streaming kernels).
//
// Method (Puro-2B report, arxiv-wiki summary, "Approach" item (4)): blockwise
// FP8 E4M3 with one fp32 scale per 1-D group of 128 activation elements or per
// 128x128 weight block. Reading of the scale (not printed on the pages):
// qscale = 448/amax, s = amax/448 (fp32, round-to-nearest-even), amax == 0 or
// an overflowing qscale gives qscale = s = 1; code = E4M3_satfinite_rn(x*qscale).
//
// One CTA of 256 threads owns a 128x128 tile of the bf16 input (32 KB).
// Thread t holds an 8x8 sub-block: rows 8*(t/16) .. +7, columns 8*(t%16) .. +7,
// read as eight 16-byte vectors (each warp instruction reads two full 256-byte
// row segments). From the registers it derives
//   * row groups (1x128): the 16 threads of a half-warp share a row, so the
//     amax is a 4-step xor shuffle;
//   * column groups (128x1): per-thread max over its 8 rows, a shuffle with the
//     other half-warp, then a 8-warp reduction through shared memory;
//   * the 128x128 block amax: a warp reduction plus the same 8-warp step.
// Row codes go out as 8-byte stores (16 lanes cover a 128-byte row segment);
// transposed codes as 8-byte stores of 8 consecutive tokens of one column.
// Nothing is staged through global memory; scratch is 4.5 KB of shared memory.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace fp8bw {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;

enum QuantMode : int {
  kModeRow = 0,    // row-wise codes + scales
  kModeCol = 1,    // transposed column-wise codes + scales
  kModeRowCol = 2, // both, one read of the input
  kModeBlock = 3,  // 128x128 block scale; codes row-major and optionally transposed
};

struct QuantArgs {
  const uint16_t* x;
  int64_t rows, cols;
  uint8_t* q_row;   // [rows, cols]  (block mode: q)
  float* s_row;     // [ceil(cols/128)][rows]
  uint8_t* q_col;   // [cols, rows]  (block mode: q_t, may be null)
  float* s_col;     // [ceil(rows/128)][cols]
  float* s_block;   // [ceil(rows/128)][ceil(cols/128)]
};

__device__ __forceinline__ float bf16_lo(uint32_t w) {
  return __uint_as_float(w << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t w) {
  return __uint_as_float(w & 0xFFFF0000u);
}

// qscale / s pair of a group (see the file comment).
__device__ __forceinline__ void group_scale(float amax, float& qscale,
                                            float& s) {
  float q = __fdiv_rn(448.0f, amax);
  if (amax == 0.0f || !isfinite(q)) {
    qscale = 1.0f;
    s = 1.0f;
  } else {
    qscale = q;
    s = __fdiv_rn(amax, 448.0f);
  }
}

// Two fp32 values -> two E4M3 codes (round to nearest even, satfinite);
// `a` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// Encode 8 values (already multiplied by qscale) into 8 bytes.
__device__ __forceinline__ uint2 pack8(const float (&t)[8]) {
  uint2 r;
  r.x = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
  r.y = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
  return r;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads) quant_tile_kernel(QuantArgs a) {
  __shared__ __align__(16) float red[kThreads / 32][kTile];  // per-warp column maxima
  __shared__ __align__(16) float colq[kTile];                // column qscales
  __shared__ float blk[kThreads / 32];

  const int t = threadIdx.x;
  const int warp = t >> 5;
  const int lane = t & 31;
  const int rb = t >> 4;   // 0..15: rows 8*rb .. 8*rb+7 of the tile
  const int cg = t & 15;   // 0..15: columns 8*cg .. 8*cg+7 of the tile

  const int64_t rows = a.rows, cols = a.cols;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTile + rb * 8;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTile + cg * 8;
  // rows and cols are multiples of 16: an 8-wide run is all in or all out.
  const bool cvalid = c0 < cols;
  const bool rvalid = r0 < rows;

  // ---- load the 8x8 sub-block as packed bf16 pairs (zeros outside) --------
  uint32_t v[8][4];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (cvalid && rvalid)
      w = __ldcs(reinterpret_cast<const uint4*>(a.x + (r0 + p) * cols + c0));
    v[p][0] = w.x;
    v[p][1] = w.y;
    v[p][2] = w.z;
    v[p][3] = w.w;
  }

  if constexpr (MODE == kModeBlock) {
    // ---- one amax for the whole 128x128 block ------------------------------
    float m = 0.0f;
#pragma unroll
    for (int p = 0; p < 8; ++p)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        m = fmaxf(m, fmaxf(fabsf(bf16_lo(v[p][j])), fabsf(bf16_hi(v[p][j]))));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) blk[warp] = m;
    __syncthreads();
    float amax = blk[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, blk[w]);
    float qs, s;
    group_scale(amax, qs, s);
    if (t == 0) {
      const int64_t nkb = (cols + kTile - 1) / kTile;
      a.s_block[static_cast<int64_t>(blockIdx.y) * nkb + blockIdx.x] = s;
    }
    if (cvalid && rvalid) {
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        float tv[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tv[2 * j] = __fmul_rn(bf16_lo(v[p][j]), qs);
          tv[2 * j + 1] = __fmul_rn(bf16_hi(v[p][j]), qs);
        }
        *reinterpret_cast<uint2*>(a.q_row + (r0 + p) * cols + c0) = pack8(tv);
      }
      if (a.q_col != nullptr) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float tv[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const float x = (j & 1) ? bf16_hi(v[p][j >> 1]) : bf16_lo(v[p][j >> 1]);
            tv[p] = __fmul_rn(x, qs);
          }
          *reinterpret_cast<uint2*>(a.q_col + (c0 + j) * rows + r0) = pack8(tv);
        }
      }
    }
    return;
  } else {
    if constexpr (MODE == kModeRow || MODE == kModeRowCol) {
      // ---- row groups: 16 lanes of a half-warp share each row --------------
      float srow[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          m = fmaxf(m, fmaxf(fabsf(bf16_lo(v[p][j])), fabsf(bf16_hi(v[p][j]))));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1)
          m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        float qs, s;
        group_scale(m, qs, s);
        srow[p] = s;
        if (cvalid && rvalid) {
          float tv[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tv[2 * j] = __fmul_rn(bf16_lo(v[p][j]), qs);
            tv[2 * j + 1] = __fmul_rn(bf16_hi(v[p][j]), qs);
          }
          *reinterpret_cast<uint2*>(a.q_row + (r0 + p) * cols + c0) = pack8(tv);
        }
      }
      if (cg == 0 && rvalid && blockIdx.x * kTile < cols) {
        float* dst = a.s_row + static_cast<int64_t>(blockIdx.x) * rows + r0;
        reinterpret_cast<float4*>(dst)[0] =
            make_float4(srow[0], srow[1], srow[2], srow[3]);
        reinterpret_cast<float4*>(dst)[1] =
            make_float4(srow[4], srow[5], srow[6], srow[7]);
      }
    }

    if constexpr (MODE == kModeCol || MODE == kModeRowCol) {
      // ---- column groups: 8 rows here, x2 across the half-warps, x8 warps --
      float cm[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float lo = 0.0f, hi = 0.0f;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          lo = fmaxf(lo, fabsf(bf16_lo(v[p][j])));
          hi = fmaxf(hi, fabsf(bf16_hi(v[p][j])));
        }
        cm[2 * j] = lo;
        cm[2 * j + 1] = hi;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        cm[j] = fmaxf(cm[j], __shfl_xor_sync(0xFFFFFFFFu, cm[j], 16));
      if (lane < 16) {
        float4* dst = reinterpret_cast<float4*>(&red[warp][cg * 8]);
        dst[0] = make_float4(cm[0], cm[1], cm[2], cm[3]);
        dst[1] = make_float4(cm[4], cm[5], cm[6], cm[7]);
      }
      __syncthreads();
      if (t < kTile) {
        float m = red[0][t];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w][t]);
        float qs, s;
        group_scale(m, qs, s);
        colq[t] = qs;
        const int64_t col = static_cast<int64_t>(blockIdx.x) * kTile + t;
        if (col < cols && static_cast<int64_t>(blockIdx.y) * kTile < rows)
          a.s_col[static_cast<int64_t>(blockIdx.y) * cols + col] = s;
      }
      __syncthreads();
      if (cvalid && rvalid) {
        const float4 q0 = *reinterpret_cast<const float4*>(&colq[cg * 8]);
        const float4 q1 = *reinterpret_cast<const float4*>(&colq[cg * 8 + 4]);
        const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float tv[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const float x = (j & 1) ? bf16_hi(v[p][j >> 1]) : bf16_lo(v[p][j >> 1]);
            tv[p] = __fmul_rn(x, qv[j]);
          }
          *reinterpret_cast<uint2*>(a.q_col + (c0 + j) * rows + r0) = pack8(tv);
        }
      }
    }
  }
}

}  // namespace

// Launchers (shapes and pointers already validated by the C ABI layer).
cudaError_t launch_quantize(int mode, const uint16_t* x, int64_t rows,
                            int64_t cols, uint8_t* q_row, float* s_row,
                            uint8_t* q_col, float* s_col, float* s_block,
                            cudaStream_t stream) {
  QuantArgs a{x, rows, cols, q_row, s_row, q_col, s_col, s_block};
  dim3 grid(static_cast<unsigned>((cols + kTile - 1) / kTile),
            static_cast<unsigned>((rows + kTile - 1) / kTile));
  switch (mode) {
    case kModeRow:
      quant_tile_kernel<kModeRow><<<grid, kThreads, 0, stream>>>(a);
      break;
    case kModeCol:
      quant_tile_kernel<kModeCol><<<grid, kThreads, 0, stream>>>(a);
      break;
    case kModeRowCol:
      quant_tile_kernel<kModeRowCol><<<grid, kThreads, 0, stream>>>(a);
      break;
    default:
      quant_tile_kernel<kModeBlock><<<grid, kThreads, 0, stream>>>(a);
      break;
  }
  return cudaGetLastError();
}

}  // namespace fp8bw
