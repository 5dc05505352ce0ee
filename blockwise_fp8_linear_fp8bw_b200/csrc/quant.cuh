// quant.cuh -- E4M3 quantisers for sm_100a (HBM-bound streaming kernels).
//
// Method (Puro-2B report, arxiv-wiki summary, "Approach" item (4)): blockwise
// FP8 E4M3 with one fp32 scale per 1-D group of 128 activation elements or per
// 128x128 weight block. Reading of the scale (not printed on the pages):
// qscale = 448/amax, s = amax/448 (fp32, round-to-nearest-even), amax == 0 or
// an overflowing qscale gives qscale = s = 1; code = E4M3_satfinite_rn(x*qscale).
//
// One persistent kernel, several modes. Each CTA (256 threads, two per SM)
// walks 128x128 tiles of the bf16 input; the next two tiles are fetched by TMA
// into a double-buffered shared-memory ring while the current one is worked
// on, so HBM reads stay in flight across the whole kernel.
// Thread t owns an 8x8 sub-block of the tile: rows 8*(t/16) .. +7, columns
// 8*(t%16) .. +7, read from shared memory as eight 16-byte vectors. From the
// registers it derives
//   * row groups (1x128): the 16 threads of a half-warp share 8 rows; the
//     amax is a packed-bf16 max and a 4-step xor shuffle, each row's two
//     divisions are done once (by one lane of the half-warp) and the qscale
//     broadcast; codes leave as 8-byte stores (a half-warp writes one
//     128-byte row segment), scales through shared memory as one 512-byte
//     run;
//   * column groups (128x1): per-thread max over its 8 rows, a shuffle with
//     the other half-warp, then an 8-warp reduction through shared memory; the
//     transposed codes (8 tokens of one column = 8 bytes per thread) go to a
//     128x128-byte shared tile, 8-byte units xor-swizzled by column block so
//     the writes are bank-conflict free, and leave as coalesced 16-byte rows;
//   * the 128x128 block amax (weights): a warp reduction plus the 8-warp step.
// Shared memory per CTA: 64 KB input ring + 16 KB transposed codes + 5 KB.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstring>

#include "common.cuh"

namespace fp8bw {

namespace {

constexpr int kQTile = 128;
constexpr int kQThreads = 256;
constexpr int kQTileBytes = kQTile * kQTile * 2;  // one bf16 input tile

enum QuantMode : int {
  kModeRow = 0,     // row-wise codes + scales
  kModeCol = 1,     // transposed column-wise codes + scales
  kModeRowCol = 2,  // both, one read of the input
  kModeBlock = 3,   // 128x128 block scale; codes row-major and optionally transposed
};

struct QuantArgs {
  int64_t rows, cols;
  int tiles_r, tiles_c;
  uint8_t* q_row;   // [rows, cols]  (block mode: q)
  float* s_row;     // [ceil(cols/128)][rows]
  uint8_t* q_col;   // [cols, rows]  (block mode: q_t, may be null)
  float* s_col;     // [ceil(rows/128)][cols]
  float* s_block;   // [ceil(rows/128)][ceil(cols/128)]
};

// One launch quantises up to kMaxQuantJobs tensors ("jobs") in the same mode:
// their 128x128 tiles are numbered one after another (job j owns tiles
// [tile_end[j-1], tile_end[j])) and the persistent CTAs walk the combined
// range, so small tensors share one launch's ramp and tail.
constexpr int kMaxQuantJobs = 8;

struct QuantJobs {
  CUtensorMap maps[kMaxQuantJobs];   // bf16 input of each job
  QuantArgs args[kMaxQuantJobs];
  int tile_end[kMaxQuantJobs];       // cumulative tile counts
  int count;
};

struct QuantSmem {
  static constexpr int kIn = 0;                                 // 2 x 32 KB
  static constexpr int kT = 2 * kQTileBytes;                    // 16 KB
  static constexpr int kRed = kT + kQTile * kQTile;             // 8 x 128 floats
  static constexpr int kColQ = kRed + 8 * kQTile * 4;           // 128 floats
  static constexpr int kSRow = kColQ + kQTile * 4;              // 128 floats
  static constexpr int kBlk = kSRow + kQTile * 4;               // 8 floats
  static constexpr int kBar = kBlk + 64;                        // 2 mbarriers
  static constexpr int kFlag = kBar + 16;
  static constexpr int kBytes = kFlag + 16;
  static constexpr int kAlloc = kBytes + 128;                   // base aligned to 128
};

// Encode 8 values (already multiplied by qscale) into 8 bytes.
__device__ __forceinline__ uint2 pack8(const float (&t)[8]) {
  uint2 r;
  r.x = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
  r.y = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
  return r;
}

// Byte offset, in the transposed tile T[col][token], of the 8-byte unit that
// holds tokens 8*u .. 8*u+7 of column k: the unit index is xor-ed with the
// column block k/8, so the 16 column blocks of a half-warp hit 16 different
// bank pairs.
__device__ __forceinline__ int t_unit_offset(int k, int u) {
  return k * kQTile + ((u ^ (k >> 3)) & 15) * 8;
}

template <int MODE, bool POW2>
__global__ void __launch_bounds__(kQThreads, 2)
    quant_tile_kernel(const __grid_constant__ QuantJobs jobs) {
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(qsmem_raw) + 127) & ~static_cast<uintptr_t>(127));
  using S = QuantSmem;
  float(*red)[kQTile] = reinterpret_cast<float(*)[kQTile]>(smem + S::kRed);
  float* colq = reinterpret_cast<float*>(smem + S::kColQ);
  float* srow_s = reinterpret_cast<float*>(smem + S::kSRow);
  float* blk = reinterpret_cast<float*>(smem + S::kBlk);
  uint8_t* T = smem + S::kT;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + S::kBar;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + S::kFlag);

  const int t = threadIdx.x;
  const int warp = t >> 5;
  const int lane = t & 31;
  const int rb = t >> 4;   // 0..15: rows 8*rb .. 8*rb+7 of the tile
  const int cg = t & 15;   // 0..15: columns 8*cg .. 8*cg+7 of the tile
  const int num_tiles = jobs.tile_end[jobs.count - 1];
  // The job that owns combined tile `tile`.
  auto job_of = [&](int tile) {
    int j = 0;
    while (j + 1 < jobs.count && tile >= jobs.tile_end[j]) ++j;
    return j;
  };
  // TMA load of combined tile `tile` into input buffer `b`.
  auto load_tile = [&](int tile, int b) {
    const int j = job_of(tile);
    const int lt = tile - (j > 0 ? jobs.tile_end[j - 1] : 0);
    const int tcs = jobs.args[j].tiles_c;
    mbar_arrive_expect_tx(bar0 + 8u * b, kQTileBytes);
    tma_load_2d(sbase + S::kIn + b * kQTileBytes, &jobs.maps[j], bar0 + 8u * b,
                (lt % tcs) * kQTile, (lt / tcs) * kQTile);
  };

  if (t == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    *abort_flag = 0u;
    fence_mbar_init();
    for (int j = 0; j < jobs.count; ++j) prefetch_tmap(&jobs.maps[j]);
  }
  __syncthreads();
  // Set-up done: let the next kernel be scheduled, and wait for the previous
  // one before any global memory is read or written.
  launch_dependents();
  grid_dependency_wait();
  // Thread 0 keeps, per input buffer, the phase parity of a load it issued and
  // that nobody has waited for yet (-1: none).
  int pend[2] = {-1, -1};
  if (t == 0) {
    for (int k = 0; k < 2; ++k) {
      const int tile = blockIdx.x + k * gridDim.x;
      if (tile < num_tiles) {
        load_tile(tile, k);
        pend[k] = 0;
      }
    }
  }

  int k = 0;
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++k) {
    const int buf = k & 1;
    const bool got = mbar_wait(bar0 + 8u * buf, (k >> 1) & 1, abort_flag, kErrTimeoutTma);
    if (!__syncthreads_and(got ? 1 : 0)) break;
    pend[buf] = -1;
    const int job = job_of(tile);
    const QuantArgs& a = jobs.args[job];
    const int64_t rows = a.rows, cols = a.cols;
    const int lt = tile - (job > 0 ? jobs.tile_end[job - 1] : 0);
    const int tr = lt / a.tiles_c, tc = lt % a.tiles_c;
    const int64_t r0 = static_cast<int64_t>(tr) * kQTile + rb * 8;
    const int64_t c0 = static_cast<int64_t>(tc) * kQTile + cg * 8;
    // rows and cols are multiples of 16: an 8-wide run is all in or all out.
    const bool cvalid = c0 < cols;
    const bool rvalid = r0 < rows;

    // ---- the 8x8 sub-block from shared memory (zeros outside the tensor) --
    uint32_t v[8][4];
    {
      const uint16_t* in = reinterpret_cast<const uint16_t*>(smem + S::kIn + buf * kQTileBytes);
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const uint4 w = *reinterpret_cast<const uint4*>(in + (rb * 8 + p) * kQTile + cg * 8);
        v[p][0] = w.x;
        v[p][1] = w.y;
        v[p][2] = w.z;
        v[p][3] = w.w;
      }
    }
    __syncthreads();  // the input buffer is free: fetch the tile after next
    if (t == 0) {
      const int next = tile + 2 * gridDim.x;
      if (next < num_tiles) {
        load_tile(next, buf);
        pend[buf] = ((k >> 1) + 1) & 1;
      }
    }

    if constexpr (MODE == kModeBlock) {
      // ---- one amax for the whole 128x128 block -----------------------------
      uint32_t m2 = 0u;
#pragma unroll
      for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j) m2 = max_bf16x2(m2, abs_bf16x2(v[p][j]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m2 = max_bf16x2(m2, __shfl_xor_sync(0xFFFFFFFFu, m2, o));
      const float m = max_halves(m2);
      if (lane == 0) blk[warp] = m;
      __syncthreads();
      float amax = blk[0];
#pragma unroll
      for (int w = 1; w < kQThreads / 32; ++w) amax = fmaxf(amax, blk[w]);
      float qs, s;
      scale_of<POW2>(amax, qs, s);
      if (t == 0) a.s_block[static_cast<int64_t>(tr) * a.tiles_c + tc] = s;
      if (cvalid && rvalid) {
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          float tv[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) scale_pair(v[p][j], qs, tv[2 * j], tv[2 * j + 1]);
          *reinterpret_cast<uint2*>(a.q_row + (r0 + p) * cols + c0) = pack8(tv);
        }
      }
      if (a.q_col != nullptr) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float tv[8];
#pragma unroll
          for (int p = 0; p < 8; p += 2) {
            const float x0 = (j & 1) ? bf16_hi(v[p][j >> 1]) : bf16_lo(v[p][j >> 1]);
            const float x1 = (j & 1) ? bf16_hi(v[p + 1][j >> 1]) : bf16_lo(v[p + 1][j >> 1]);
            fmul2(tv[p], tv[p + 1], x0, x1, qs, qs);
          }
          *reinterpret_cast<uint2*>(T + t_unit_offset(cg * 8 + j, rb)) = pack8(tv);
        }
      }
    } else {
      if constexpr (MODE == kModeRow || MODE == kModeRowCol) {
        // ---- row groups: the 16 lanes of a half-warp share rows 8rb..8rb+7.
        // amax by packed bf16 max + xor shuffles (every lane gets all 8);
        // lane (cg & 7) then computes the two divisions of row (cg & 7) and
        // the qscales are broadcast back by shuffle.
        float my_amax = 0.0f;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          uint32_t m2 = max_bf16x2(max_bf16x2(abs_bf16x2(v[p][0]), abs_bf16x2(v[p][1])),
                                   max_bf16x2(abs_bf16x2(v[p][2]), abs_bf16x2(v[p][3])));
#pragma unroll
          for (int o = 8; o > 0; o >>= 1)
            m2 = max_bf16x2(m2, __shfl_xor_sync(0xFFFFFFFFu, m2, o));
          const float am = max_halves(m2);
          if ((cg & 7) == p) my_amax = am;
        }
        float my_qs, my_s;
        scale_of<POW2>(my_amax, my_qs, my_s);
        if (cg < 8) srow_s[rb * 8 + cg] = my_s;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float qs = __shfl_sync(0xFFFFFFFFu, my_qs, (lane & 16) | p);
          if (cvalid && rvalid) {
            float tv[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) scale_pair(v[p][j], qs, tv[2 * j], tv[2 * j + 1]);
            *reinterpret_cast<uint2*>(a.q_row + (r0 + p) * cols + c0) = pack8(tv);
          }
        }
      }

      if constexpr (MODE == kModeCol || MODE == kModeRowCol) {
        // ---- column groups: 8 rows here, x2 across the half-warps, x8 warps
        float cm[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t m2 = abs_bf16x2(v[0][j]);
#pragma unroll
          for (int p = 1; p < 8; ++p) m2 = max_bf16x2(m2, abs_bf16x2(v[p][j]));
          m2 = max_bf16x2(m2, __shfl_xor_sync(0xFFFFFFFFu, m2, 16));
          cm[2 * j] = bf16_lo(m2);
          cm[2 * j + 1] = bf16_hi(m2);
        }
        if (lane < 16) {
          float4* dst = reinterpret_cast<float4*>(&red[warp][cg * 8]);
          dst[0] = make_float4(cm[0], cm[1], cm[2], cm[3]);
          dst[1] = make_float4(cm[4], cm[5], cm[6], cm[7]);
        }
        __syncthreads();
        if (t < kQTile) {
          float m = red[0][t];
#pragma unroll
          for (int w = 1; w < kQThreads / 32; ++w) m = fmaxf(m, red[w][t]);
          float qs, s;
          scale_of<POW2>(m, qs, s);
          colq[t] = qs;
          const int64_t col = static_cast<int64_t>(tc) * kQTile + t;
          if (col < cols) a.s_col[static_cast<int64_t>(tr) * cols + col] = s;
        }
        __syncthreads();
        const float4 q0 = *reinterpret_cast<const float4*>(&colq[cg * 8]);
        const float4 q1 = *reinterpret_cast<const float4*>(&colq[cg * 8 + 4]);
        const float qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float tv[8];
#pragma unroll
          for (int p = 0; p < 8; p += 2) {
            const float x0 = (j & 1) ? bf16_hi(v[p][j >> 1]) : bf16_lo(v[p][j >> 1]);
            const float x1 = (j & 1) ? bf16_hi(v[p + 1][j >> 1]) : bf16_lo(v[p + 1][j >> 1]);
            fmul2(tv[p], tv[p + 1], x0, x1, qv[j], qv[j]);
          }
          *reinterpret_cast<uint2*>(T + t_unit_offset(cg * 8 + j, rb)) = pack8(tv);
        }
      }
    }

    __syncthreads();  // T (and the row scales) complete
    if constexpr (MODE == kModeRow || MODE == kModeRowCol) {
      // row scales: one 512-byte run s_row[tc][tr*128 .. +127]
      if (t < kQTile / 4) {
        const int64_t row = static_cast<int64_t>(tr) * kQTile + t * 4;
        if (row < rows)
          *reinterpret_cast<float4*>(a.s_row + static_cast<int64_t>(tc) * rows + row) =
              *reinterpret_cast<const float4*>(&srow_s[t * 4]);
      }
    }
    if (MODE == kModeCol || MODE == kModeRowCol || (MODE == kModeBlock && a.q_col != nullptr)) {
      // transposed codes: column k of the tile is 128 contiguous tokens of
      // q_col row (tc*128 + k); 8 threads write one 128-byte row, 16 bytes each.
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int idx = it * kQThreads + t;   // 0..1023
        const int kk = idx >> 3;              // tile column
        const int ch = idx & 7;               // 16-byte chunk = units 2ch, 2ch+1
        const int64_t col = static_cast<int64_t>(tc) * kQTile + kk;
        const int64_t tok = static_cast<int64_t>(tr) * kQTile + ch * 16;
        if (col < cols && tok < rows) {
          const uint2 lo = *reinterpret_cast<const uint2*>(T + t_unit_offset(kk, 2 * ch));
          const uint2 hi = *reinterpret_cast<const uint2*>(T + t_unit_offset(kk, 2 * ch + 1));
          *reinterpret_cast<uint4*>(a.q_col + col * rows + tok) = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
      }
    }
    __syncthreads();  // T and the scale staging may be reused
  }

  if (t == 0) {
    // After an expired wait the loop ends early: let the copies already issued
    // land before the shared memory is released (bounded as well).
    for (int b = 0; b < 2; ++b) {
      if (pend[b] < 0) continue;
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar0 + 8u * b, static_cast<uint32_t>(pend[b])) &&
             globaltimer_ns() - t0 < kWaitLimitNs) {
      }
    }
  }
}

}  // namespace

// 2-D bf16 tensor [rows, cols] read in 128 x 128 boxes (256-byte rows, no
// swizzle); out-of-range elements read as zero.
int encode_bf16_in(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows);

// One quantisation job of a launch (shapes and pointers already validated
// by the C ABI layer).
struct QuantJob {
  const uint16_t* x;
  int64_t rows, cols;
  uint8_t* q_row;
  float* s_row;
  uint8_t* q_col;
  float* s_col;
  float* s_block;
};

// Launch one kernel over 1..kMaxQuantJobs jobs of the same mode.
int launch_quantize_jobs(int mode, bool pow2, const QuantJob* jb, int count, int device,
                         int sm_count, cudaStream_t stream) {
  if (count < 1 || count > kMaxQuantJobs) return FP8BW_ERR_SHAPE;
  QuantJobs jobs;
  memset(&jobs, 0, sizeof jobs);
  int64_t tiles = 0;
  for (int i = 0; i < count; ++i) {
    QuantArgs& a = jobs.args[i];
    a = QuantArgs{jb[i].rows, jb[i].cols, static_cast<int>((jb[i].rows + kQTile - 1) / kQTile),
                  static_cast<int>((jb[i].cols + kQTile - 1) / kQTile), jb[i].q_row, jb[i].s_row,
                  jb[i].q_col, jb[i].s_col, jb[i].s_block};
    const int st = encode_bf16_in(&jobs.maps[i], jb[i].x, static_cast<uint64_t>(jb[i].cols),
                                  static_cast<uint64_t>(jb[i].rows));
    if (st != FP8BW_OK) return st;
    tiles += static_cast<int64_t>(a.tiles_r) * a.tiles_c;
    if (tiles > INT32_MAX) return FP8BW_ERR_SHAPE;
    jobs.tile_end[i] = static_cast<int>(tiles);
  }
  jobs.count = count;
  if (tiles == 0) return FP8BW_OK;
  const int grid = static_cast<int>(tiles < 2 * sm_count ? tiles : 2 * sm_count);
  using Kernel = void (*)(QuantJobs);
  static const Kernel kernels[8] = {
      quant_tile_kernel<kModeRow, false>,    quant_tile_kernel<kModeCol, false>,
      quant_tile_kernel<kModeRowCol, false>, quant_tile_kernel<kModeBlock, false>,
      quant_tile_kernel<kModeRow, true>,     quant_tile_kernel<kModeCol, true>,
      quant_tile_kernel<kModeRowCol, true>,  quant_tile_kernel<kModeBlock, true>};
  static DevicePrep prep;
  int unused = 0;
  const int pst = prepare_for_device(prep, device, &unused, [&](int*) {
    for (Kernel k : kernels)
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               QuantSmem::kAlloc) != cudaSuccess)
        return static_cast<int>(FP8BW_ERR_LAUNCH);
    return static_cast<int>(FP8BW_OK);
  });
  if (pst != FP8BW_OK) return pst;
  const Kernel kernel = kernels[(mode >= 0 && mode < 4 ? mode : kModeBlock) + (pow2 ? 4 : 0)];
  if (launch_kernel(kernel, dim3(grid), dim3(kQThreads), QuantSmem::kAlloc, stream, jobs) !=
      cudaSuccess)
    return FP8BW_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? FP8BW_OK : FP8BW_ERR_LAUNCH;
}

// Launch for one tensor.
int launch_quantize(int mode, bool pow2, const uint16_t* x, int64_t rows, int64_t cols,
                    uint8_t* q_row, float* s_row, uint8_t* q_col, float* s_col, float* s_block,
                    int device, int sm_count, cudaStream_t stream) {
  const QuantJob job{x, rows, cols, q_row, s_row, q_col, s_col, s_block};
  return launch_quantize_jobs(mode, pow2, &job, 1, device, sm_count, stream);
}

}  // namespace fp8bw
